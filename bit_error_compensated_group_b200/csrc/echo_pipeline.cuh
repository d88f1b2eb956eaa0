// echo_pipeline.cuh -- bulk-copy (TMA) staged versions of the two kernels
// that stream the inputs and the EMA state.
//
// Why: each element of the quantize and reduce passes moves 18 bytes of
// input/state (bf16 x, two fp32 EMAs, read) before any math can start. With
// loads issued from registers, bytes in flight per SM are capped by the
// register file; here one producer lane per CTA streams whole tiles
// (T groups x (bf16 x, e_long, e_short)) into a ring of shared-memory stages
// with cp.async.bulk (the TMA engine, 1-D, no tensor map, this CTA only), and
// the consumer warps compute from shared memory and write results straight
// back to HBM. Several 20 KB tiles per CTA are in flight at any time.
//
// Synchronization per stage: full[s] (producer arrive + transaction bytes)
// and empty[s] (one arrive per consumer warp). Every wait is bounded by a
// wall-clock limit (Args::wait_ns, the handle's setting, 1 s by default):
// on expiry the kernel sets ECHO_FLAG_TIMEOUT, stops, and the producer lane
// waits (again bounded) for the copies it issued before the CTA exits. Partial last groups (not 16-byte sized) take the direct
// register path of echo_kernels.cuh.
#pragma once

#include "echo_kernels.cuh"

namespace echo_dev {

constexpr int kConsumerWarps = 8;
constexpr int kPipeThreads = (kConsumerWarps + 1) * 32;
constexpr int kTileElems = kConsumerWarps * 32 * 8;           // 2048 elements per tile
constexpr int kStageBytes = kTileElems * (2 + 4 + 4);          // bf16 x + two fp32 EMAs
// ring stages per pipelined kernel (with and without feedback), measured on
// B200: fewer tiles in flight per CTA stream faster here. The quantize pass
// with feedback keeps each slot one tile longer (until the bulk stores of the
// EMAs have read it).
constexpr int kStagesQuantizeFB = 3;
constexpr int kStagesReduceFB = 4;
constexpr int kStagesQuantizeNF = 4;
constexpr int kStagesReduceNF = 4;
// dynamic shared memory of a pipelined kernel with NS ring stages
__host__ __device__ constexpr int pipe_smem(int NS) { return NS * kStageBytes + 2 * NS * 8 + 16; }

// ------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Programmatic dependent launch. The quantize pass lets the owners' pass
// launch as soon as every quantize CTA has started; the owners' consumers wait
// for the quantize grid to complete (and its writes to be visible) before they
// read the all-to-all payload. Without a programmatic dependency the wait
// returns at once.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy shared -> global (this CTA's buffer); dst, src, bytes multiples of 16
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_addr(src)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Hint: bring [src, src + bytes) into L2 (address 16-byte aligned, bytes a
// multiple of 16). Nothing waits on it.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------ tile walk

// A run is a contiguous range of full groups [j0, j1) of one rank, clipped to
// the call's group-column window [c0, c1). The tile sequence of a kernel is
// the concatenation of its runs cut into tiles of at most T groups. The
// cursor walks it monotonically (tile indices only grow).
struct Tile {
    int rank;
    long long j0;
    int count;
};

template <int GROUP, int M, bool RK, int KIND>
struct RunWalker {
    static constexpr int T = M * kTileElems / GROUP;   // groups per tile (M sub-tiles)
    // KIND 0: non-owned runs of the ranks [rank_lo, rank_hi) (quantize);
    // KIND 1: the owned runs of those ranks (reduce). RK: one rank of a
    // multi-GPU call (rank_hi = rank_lo + 1), whose calls may be chunked.
    // G, P and the window are read from the kernel arguments when needed
    // rather than held in registers.
    int run;            // current run index
    long long base;     // first tile index of the current run
    long long run_j0, run_len;

    // run `run` before clipping. KIND 0, rank r = run / 2: [0, lo) for even
    // runs, [hi, G) for odd; KIND 1: [lo, hi) of rank `run`, where [lo, hi)
    // is that rank's owned segment. In a chunked rank call (chunk_k > 0)
    // KIND 0 has a run per owner s = run - P rank_lo: owner s's part of the
    // chunk, empty for the rank's own segment; KIND 1 the owned segment's
    // part. Clipped to the call's full-group window [c0, c1) (a partial last
    // group takes the kernels' scalar path).
    __device__ __forceinline__ void load_run(const Args& a) {
        long long b, e;
        if (RK && a.chunk_k > 0) {
            const int s = KIND == 0 ? run - a.P * a.rank_lo : run;
            segment_part(a, s, &b, &e);
            if (KIND == 0 && s == a.rank_lo) e = b;
        } else {
            const int r = KIND == 0 ? run >> 1 : run;
            const long long lo = (long long)r * a.G / a.P, hi = (long long)(r + 1) * a.G / a.P;
            if (KIND == 1) {
                b = lo;
                e = hi;
            } else if ((run & 1) == 0) {
                b = 0;
                e = lo;
            } else {
                b = hi;
                e = a.G;
            }
        }
        b = max(b, a.c0);
        e = min(e, a.c1);
        run_j0 = b;
        run_len = max(0LL, e - b);
    }
    __device__ __forceinline__ int runs_per_rank(const Args& a) const {
        return KIND == 1 ? 1 : ((RK && a.chunk_k > 0) ? a.P : 2);
    }
    __device__ __forceinline__ int runs(const Args& a) const { return runs_per_rank(a) * a.rank_hi; }
    __device__ __forceinline__ int rank_of_run(const Args& a) const {
        return RK ? a.rank_lo : (KIND == 0 ? (run >> 1) : run);
    }

    __device__ __forceinline__ explicit RunWalker(const Args& a) : base(0) {
        run = runs_per_rank(a) * a.rank_lo;
        if (run < runs(a)) load_run(a);
    }

    // Tile k (k never decreases between calls); false when past the end.
    __device__ __forceinline__ bool locate(long long k, Tile* t, const Args& a) {
        while (run < runs(a)) {
            const long long nt = (run_len + T - 1) / T;
            if (k < base + nt) {
                const long long off = (k - base) * T;
                t->rank = rank_of_run(a);
                t->j0 = run_j0 + off;
                t->count = (int)min((long long)T, run_len - off);
                return true;
            }
            base += nt;
            ++run;
            if (run < runs(a)) load_run(a);
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

template <int NS>
__device__ __forceinline__ PipeShared pipe_shared(uint8_t* smem) {
    PipeShared p;
    p.stages = smem;
    p.full = reinterpret_cast<uint64_t*>(smem + NS * kStageBytes);
    p.empty = p.full + NS;
    p.abort = reinterpret_cast<volatile int*>(p.empty + NS);
    return p;
}

// `consumers`: the warps that release each stage (all consumer warps, or one
// half of them when the halves take alternate tiles)
template <int NS>
__device__ __forceinline__ void pipe_init(const PipeShared& p, int consumers = kConsumerWarps) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&p.full[s], 1);
            mbar_init(&p.empty[s], consumers);
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
// adds the two EMA tiles of the tile's rank (then M == 1); without state a
// stage holds M = 5 sub-tiles of bf16 inputs, the same 20 KB.
// PF_CB > 0 (the owners' pass of one rank of a multi-GPU call: code bytes per
// group): with each tile, also prefetch into L2 the received payload rows the
// consumers will load for it, so their plain loads of the P - 1 incoming
// slots find them there (measured on one B200: that pass 0.333 -> 0.316 ms
// on the 1 GB P = 8 message; the simulation's owners' pass, whose output
// stores keep the memory system busier, ran 3.54 -> 3.78 ms with it and goes
// without). Every source here is this GPU's own memory (see a2a_slot_t):
// the loads are plain bulk copies, none with cluster multicast.
template <int GROUP, int M, int NS, bool RK, int KIND, int PF_CB = 0>
__device__ __forceinline__ void produce(const Args& a, const PipeShared& p, RunWalker<GROUP, M, RK, KIND>& walker,
                                        bool with_state) {
    long long issued = 0;
    Tile t;
    for (long long k = blockIdx.x; walker.locate(k, &t, a); k += gridDim.x, ++issued) {
        const int s = (int)(issued % NS);
        const uint32_t use = (uint32_t)(issued / NS);
        if (issued >= NS && !mbar_wait(&p.empty[s], (use & 1u) ^ 1u, a.wait_ns, p.abort)) {
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
            const float* el = state_row_t<RK>(a, t.rank);
            bulk_load(st + kTileElems * 2, el + e0, sbytes, &p.full[s]);
            bulk_load(st + kTileElems * 6, el + a.S + e0, sbytes, &p.full[s]);
        }
        if (PF_CB > 0) {
            for (int r = 0; r < a.P; ++r) {
                if (r == t.rank) continue;
                const size_t slot = a2a_slot_t<RK>(a, r, t.j0);
                prefetch_l2(a.a2a_codes + slot * PF_CB, (uint32_t)t.count * PF_CB);
                // the parameter words, widened to 16-byte bounds (inside the
                // 256-byte aligned parameter region)
                const uintptr_t lo = reinterpret_cast<uintptr_t>(a.a2a_params + slot) & ~uintptr_t(15);
                const uintptr_t hi = (reinterpret_cast<uintptr_t>(a.a2a_params + slot + t.count) + 15) &
                                     ~uintptr_t(15);
                prefetch_l2(reinterpret_cast<const void*>(lo), (uint32_t)(hi - lo));
            }
        }
    }
    // drain: the last (up to NS) tiles' copies must land before the CTA
    // may retire, whatever happened to the consumers
    const long long first = issued > NS ? issued - NS : 0;
    for (long long i = first; i < issued; ++i) {
        const int s = (int)(i % NS);
        if (!mbar_wait(&p.full[s], (uint32_t)(i / NS) & 1u, a.wait_ns, nullptr)) {
            atomicOr(a.flags, (unsigned)ECHO_FLAG_TIMEOUT);
        }
    }
}

// ------------------------------------------------------------ packed math
//
// The tile paths compute two elements per instruction with the sm_100 paired
// binary32 operations (add/fma.rn.f32x2: each component rounds exactly like
// the scalar operation) where that cannot change a single bit:
//  * dequantization code*s + z uses one fused multiply-add: code <= 255 and
//    s is an fp16 value (11-bit significand), so code*s is exact in binary32
//    and rounding once gives the same result as multiply-then-add;
//  * a code is turned into an exact float by placing it in the mantissa of
//    2^23 (bit pattern 0x4B000000 | code) and subtracting 2^23;
//  * additions whose operands are not products (rank-ordered sums, x' - x_hat).
// Every product that the definition rounds before an addition (compensation,
// the quantizer's (v - z) * inv, both EMA terms) is a paired multiply, and
// the addition that consumes it is written fma(product, one, other) with
// `one` = 1.0 read from the kernel arguments: the assembler may fuse a paired
// multiply into a paired add that consumes it, even with an explicit .rn
// (seen on sm_100a: a tie rounded the other way), but it cannot fold a
// multiplier it does not know, and fma(p, 1, q) rounds exactly like p + q.
// Round-half-even of u in [0, 2^22) is (u + 2^23): binary32 spacing there is
// 1, so the addition itself rounds u to the nearest integer, ties to even,
// and the code sits in the low mantissa bits.
// Group min/max use min.NaN / max.NaN so that a NaN anywhere in a group
// reaches the range check.

constexpr float kMagic = 8388608.0f;   // 2^23

// Paired binary32 operations (PTX add/mul/fma.rn.f32x2).
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rr;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rr, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rr;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rr, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rr;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rr, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

// round a pair to bf16 (nearest-even); element 0 in the low half
__device__ __forceinline__ uint32_t bf16x2_rn(float2 v) {
    const __nv_bfloat162 b = __float22bfloat162_rn(v);
    return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ float nan_min(float a, float b) {
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float nan_max(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float nan_min3(float a, float b, float c) {
    float r;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float nan_max3(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Packed quantization grid of one group (same values as make_grid). A code
// decodes to code * s + z (z is the additive term zf of the scalar Grid).
struct GridP {
    float2 s, z, ns, nz, inv;
    float2 nzs;   // -zsub (nearest form)
    int C;        // 0x4B400000 - zq: signed-magic bits of code 0 (nearest and integer-zero forms)
    uint32_t param;
    bool bad;   // a value outside [-65504, 65504] or a NaN
};

// fp16 parameters of a group from its range [mn, mx] (same values as make_grid).
template <int Q, int QM>
__device__ __forceinline__ GridP grid_from_range(float mn, float mx) {
    GridP gp;
    gp.bad = !(mn >= -65504.0f && mx <= 65504.0f);
    const Grid g = group_grid<Q, QM>(__fadd_rn(mn, 0.0f), __fadd_rn(mx, 0.0f));   // -0 -> +0
    gp.s = splat(g.s);
    gp.z = splat(g.zf);
    gp.ns = splat(-g.s);
    gp.nz = splat(-g.zf);
    gp.inv = splat(g.inv);
    gp.nzs = splat(-g.zsub);
    gp.C = 0x4B400000 - g.zq;
    gp.param = g.param;
    return gp;
}

template <int L, int Q, int QM>
__device__ __forceinline__ GridP make_grid_p(float lane_min, float lane_max) {
    float mn = lane_min, mx = lane_max;
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) {
        mn = nan_min(mn, __shfl_xor_sync(kFull, mn, o));
        mx = nan_max(mx, __shfl_xor_sync(kFull, mx, o));
    }
    return grid_from_range<Q, QM>(mn, mx);
}

// p + q where p (or q) is a rounded product: fma(p, one, q), one = 1.0 at run time
__device__ __forceinline__ float2 add_after_mul2(float2 p, float2 q, const Args& a) {
    return fma2_rn(p, splat(a.one), q);
}

// 2^23 + code for a pair of values (the code sits in the low mantissa bits).
// Default form: code = round_half_even((v - z) * inv), in [0, Q] without a
// clamp because the directed parameters make [z, z + Q s] cover the group.
// Other forms: u = (v - z) * inv (nearest) or v * inv (integer zero), clamped
// to [-(Q+1), Q+1] (then rint-and-clamp agrees with clamping first); adding
// 1.5 * 2^23 rounds u to an integer with ties to even (the magic is even and
// the spacing there is 1), leaving bits 0x4B400000 + rint(u); subtracting
// C = 0x4B400000 - zq gives rint(u) + zq, clamped to [0, Q].
constexpr float kMagicSigned = 12582912.0f;   // 1.5 * 2^23

template <int QM, int Q>
__device__ __forceinline__ float2 encode2(float2 v, const GridP& g, const Args& a) {
    if (QM == kQuantDirected) {
        const float2 u = mul2_rn(add2_rn(v, g.nz), g.inv);   // (v - z) * inv
        return add_after_mul2(u, splat(kMagic), a);
    }
    float2 u = (QM == kQuantNearest) ? mul2_rn(add2_rn(v, g.nzs), g.inv) : mul2_rn(v, g.inv);
    u.x = fminf(fmaxf(u.x, -(float)(Q + 1)), (float)(Q + 1));
    u.y = fminf(fmaxf(u.y, -(float)(Q + 1)), (float)(Q + 1));
    const float2 t = add_after_mul2(u, splat(kMagicSigned), a);
    const int cx = min(max((int)__float_as_uint(t.x) - g.C, 0), Q);
    const int cy = min(max((int)__float_as_uint(t.y) - g.C, 0), Q);
    return make_float2(__uint_as_float(0x4B000000u | (uint32_t)cx), __uint_as_float(0x4B000000u | (uint32_t)cy));
}



// eight codes (2^23 + code each, in four pairs) -> packed bytes: one word at
// 4 bits, two at 8 bits. Only the low byte of each float's bit pattern is
// used; at 4 bits (hi << 4) + lo puts code 2i + 1 above code 2i without a
// carry out of the byte (both codes <= 15).
template <int BITS>
__device__ __forceinline__ uint2 pack_codes8(const float2 t[4]) {
    uint2 out;
    if (BITS == 4) {
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) b[k] = (__float_as_uint(t[k].y) << 4) + __float_as_uint(t[k].x);
        out.x = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
        out.y = 0;
    } else {
        const uint32_t p0 = __byte_perm(__float_as_uint(t[0].x), __float_as_uint(t[0].y), 0x0040);
        const uint32_t p1 = __byte_perm(__float_as_uint(t[1].x), __float_as_uint(t[1].y), 0x0040);
        const uint32_t p2 = __byte_perm(__float_as_uint(t[2].x), __float_as_uint(t[2].y), 0x0040);
        const uint32_t p3 = __byte_perm(__float_as_uint(t[3].x), __float_as_uint(t[3].y), 0x0040);
        out.x = __byte_perm(p0, p1, 0x5410);
        out.y = __byte_perm(p2, p3, 0x5410);
    }
    return out;
}

// eight packed codes (one word at 4 bits, two at 8) -> four exact float pairs
template <int BITS>
__device__ __forceinline__ void unpack_codes8(const uint32_t* w, float2 q[4]) {
    uint32_t ev[4], od[4];   // 2^23 + code of elements 2p and 2p + 1
    if (BITS == 4) {
        const uint32_t lo = w[0] & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6 in bytes 0..3
        const uint32_t hi = (w[0] >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            ev[p] = __byte_perm(lo, 0x4B000000u, 0x7650 + p);
            od[p] = __byte_perm(hi, 0x4B000000u, 0x7650 + p);
        }
    } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            ev[p] = __byte_perm(w[p >> 1], 0x4B000000u, 0x7650 + 2 * (p & 1));
            od[p] = __byte_perm(w[p >> 1], 0x4B000000u, 0x7651 + 2 * (p & 1));
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
        q[p] = add2_rn(make_float2(__uint_as_float(ev[p]), __uint_as_float(od[p])), splat(-kMagic));
}


// x' = x + eta * (w * e_short + (1 - w) * e_long), two elements
__device__ __forceinline__ float2 inject2(float2 x, float2 el, float2 es, const Args& a) {
    const float2 t = add_after_mul2(mul2_rn(splat(a.w), es), mul2_rn(splat(a.one_minus_w), el), a);
    return add_after_mul2(mul2_rn(splat(a.eta), t), x, a);
}

// e <- (1 - alpha) * e + alpha * rho, two elements
__device__ __forceinline__ float2 ema2(float2 e, float2 rho, float keep, float alpha, const Args& a) {
    return add_after_mul2(mul2_rn(splat(keep), e), mul2_rn(splat(alpha), rho), a);
}


__device__ __forceinline__ void load_f8_smem(const float* p, int c0, int c1, float2 v[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p + c0);
    const float4 b = *reinterpret_cast<const float4*>(p + c1);
    v[0] = make_float2(a.x, a.y);
    v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y);
    v[3] = make_float2(b.z, b.w);
}

__device__ __forceinline__ void store_f4_pair(float* p, float2 lo, float2 hi) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(lo.x, lo.y, hi.x, hi.y));
}

// 8 consecutive bf16 values (16 bytes) from shared memory
__device__ __forceinline__ void load_x8c_smem(const uint16_t* xs, float2 v[4]) {
    const uint4 u = *reinterpret_cast<const uint4*>(xs);
    v[0] = make_float2(bf16_lo(u.x), bf16_hi(u.x));
    v[1] = make_float2(bf16_lo(u.y), bf16_hi(u.y));
    v[2] = make_float2(bf16_lo(u.z), bf16_hi(u.z));
    v[3] = make_float2(bf16_lo(u.w), bf16_hi(u.w));
}

// 8 consecutive fp32 values to global memory in one 32-byte streaming store
// (sm_100 vector width; p must be 32-byte aligned).
__device__ __forceinline__ void store_f8_cs(float* p, const float2 v[4]) {
    asm volatile("st.global.cs.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[0].x),
                 "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), "f"(v[3].y)
                 : "memory");
}

// 8 bf16 pairs to global memory in one 32-byte streaming store (p 32-byte aligned)
__device__ __forceinline__ void store_v8_cs(void* p, uint4 lo, uint4 hi) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(lo.x), "r"(lo.y),
                 "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
                 : "memory");
}

// ------------------------------------------------------------ quantize

// One non-owned group of a tile with feedback (x, e_long, e_short staged):
// 8 consecutive elements per lane (lane t of the group's L takes elements
// [8t, 8t + 8)).
template <int GROUP, int BITS, int QM, bool RK>
__device__ __forceinline__ void quantize_tile_group(const Args& a, uint8_t* st, const Tile& t, int gi, bool act) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    const LN ln;
    const int r = t.rank;
    const long long j = t.j0 + gi;
    const int e0 = 8 * ln.t;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(st) + gi * GROUP;
    float* els = reinterpret_cast<float*>(st + kTileElems * 2) + gi * GROUP;
    float* ess = reinterpret_cast<float*>(st + kTileElems * 6) + gi * GROUP;
    float2 v[4], el[4], es[4];
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
    if (act) {
        load_x8c_smem(xs + e0, v);
        load_f8_smem(els, e0, e0 + 4, el);
        load_f8_smem(ess, e0, e0 + 4, es);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            v[p] = inject2(v[p], el[p], es[p], a);
            lmin = nan_min3(lmin, v[p].x, v[p].y);
            lmax = nan_max3(lmax, v[p].x, v[p].y);
        }
    }
    const GridP g = make_grid_p<L, Q, QM>(lmin, lmax);
    raise_flags(a, act && g.bad);
    if (!act) return;
    float2 e[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) e[p] = encode2<QM, Q>(v[p], g, a);
    uint8_t* codes = a.a2a_codes + a2a_slot_t<RK>(a, r, j) * CB;
    const uint2 pk = pack_codes8<BITS>(e);
    if (BITS == 4) *reinterpret_cast<uint32_t*>(codes + 4 * ln.t) = pk.x;
    else *reinterpret_cast<uint2*>(codes + 8 * ln.t) = pk;
    // residual x' - x_hat with x_hat = code*s + z (fused: code*s is exact)
    float2 nl[4], ns[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 rho = add2_rn(v[p], fma2_rn(add2_rn(e[p], splat(-kMagic)), g.ns, g.nz));
        nl[p] = ema2(el[p], rho, a.keep_long, a.a_long, a);
        ns[p] = ema2(es[p], rho, a.keep_short, a.a_short, a);
    }
    // the updated EMAs go back into the stage, over the values just read; the
    // warp then sends its rows to global memory with bulk stores
    *reinterpret_cast<float4*>(els + e0) = make_float4(nl[0].x, nl[0].y, nl[1].x, nl[1].y);
    *reinterpret_cast<float4*>(els + e0 + 4) = make_float4(nl[2].x, nl[2].y, nl[3].x, nl[3].y);
    *reinterpret_cast<float4*>(ess + e0) = make_float4(ns[0].x, ns[0].y, ns[1].x, ns[1].y);
    *reinterpret_cast<float4*>(ess + e0 + 4) = make_float4(ns[2].x, ns[2].y, ns[3].x, ns[3].y);
    if (ln.t == 0) a.a2a_params[a2a_slot_t<RK>(a, r, j)] = g.param;
}

// Without feedback the quantizer reads bf16 values only, and the per-group
// work (range reduction, fp16 parameters, two divisions) dominates the issue
// slots. These paths give each lane E = 16 or 32 elements (E/8 chunks of 8:
// t, t + L, t + 2L, ...) so that the group work is shared by more elements,
// and the quantizer takes the group range on packed bf16 pairs: bf16 ->
// binary32 is exact and order-preserving, so min/max on bf16 gives the same
// values. Lane minima and negated maxima travel as one bf16x2 word (min, -max),
// reduced with a single min per shuffle round (max(x) = -min(-x) exactly, and
// min.NaN keeps NaNs).
template <int GROUP, int E>
struct LaneE {
    static constexpr int L = GROUP / E;      // lanes per group
    static constexpr int GPW = 32 / L;       // groups per warp
    static constexpr int H = E / 8;          // 8-element chunks per lane
    int sub, t;
    __device__ __forceinline__ LaneE() {
        const int lane = threadIdx.x & 31;
        sub = lane / L;
        t = lane % L;
    }
    __device__ __forceinline__ int chunk(int h) const { return t + h * L; }
};

template <int GROUP>
using Lane16 = LaneE<GROUP, 16>;

constexpr int kQuantizeLaneElemsNF = 32;
constexpr int kQuantizeSubtilesNF = 4;   // 8192 elements per tile: one pass of 8 warps x 32 lanes x 32
constexpr int kReduceSubtilesNF = 4;

__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ float2 bf16_pair(uint32_t u) { return make_float2(bf16_lo(u), bf16_hi(u)); }

template <int GROUP, int BITS, int QM, bool RK>
__device__ __forceinline__ void quantize_tile_group_nf(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                       bool act) {
    using LN = LaneE<GROUP, kQuantizeLaneElemsNF>;
    constexpr int L = LN::L, H = LN::H, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    const LN ln;
    // Chunk order per group (h ^ flip): when a quarter-warp spans several
    // groups, each takes a different chunk at a time, so that the 16-byte
    // shared-memory reads of those 8 lanes fall in distinct banks (groups of
    // 32 elements at an odd index are 16 banks apart already).
    constexpr int QG = L >= 8 ? 1 : 8 / L;   // groups per quarter-warp
    const int flip = (GROUP == 32 ? (ln.sub >> 1) : (ln.sub & (QG - 1))) & (H - 1);
    const uint4* xs = reinterpret_cast<const uint4*>(st + (size_t)gi * GROUP * 2);
    uint4 w[H];
    uint32_t mm = 0x7F807F80u;   // (+inf, -(-inf)): neutral for an inactive group
    if (act) {
#pragma unroll
        for (int h = 0; h < H; ++h) w[h] = xs[ln.chunk(h ^ flip)];
        uint32_t lo = bmin2(bmin2(w[0].x, w[0].y), bmin2(w[0].z, w[0].w));
        uint32_t hi = bmax2(bmax2(w[0].x, w[0].y), bmax2(w[0].z, w[0].w));
#pragma unroll
        for (int h = 1; h < H; ++h) {
            lo = bmin2(lo, bmin2(bmin2(w[h].x, w[h].y), bmin2(w[h].z, w[h].w)));
            hi = bmax2(hi, bmax2(bmax2(w[h].x, w[h].y), bmax2(w[h].z, w[h].w)));
        }
        // (lo.even, -hi.even) and (lo.odd, -hi.odd) -> (lane min, -lane max)
        mm = bmin2(__byte_perm(lo, hi, 0x5410) ^ 0x80000000u, __byte_perm(lo, hi, 0x7632) ^ 0x80000000u);
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) mm = bmin2(mm, __shfl_xor_sync(kFull, mm, o));
    const GridP g = grid_from_range<Q, QM>(__uint_as_float(mm << 16), __uint_as_float((mm & 0xffff0000u) ^ 0x80000000u));
    raise_flags(a, act && g.bad);
    if (!act) return;
    const long long j = t.j0 + gi;
    uint8_t* codes = a.a2a_codes + a2a_slot_t<RK>(a, t.rank, j) * CB;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        float2 e[4];
        e[0] = encode2<QM, Q>(bf16_pair(w[h].x), g, a);
        e[1] = encode2<QM, Q>(bf16_pair(w[h].y), g, a);
        e[2] = encode2<QM, Q>(bf16_pair(w[h].z), g, a);
        e[3] = encode2<QM, Q>(bf16_pair(w[h].w), g, a);
        const uint2 pk = pack_codes8<BITS>(e);
        const int c = ln.chunk(h ^ flip);
        if (BITS == 4) *reinterpret_cast<uint32_t*>(codes + 4 * c) = pk.x;
        else *reinterpret_cast<uint2*>(codes + 8 * c) = pk;
    }
    if (ln.t == 0) a.a2a_params[a2a_slot_t<RK>(a, t.rank, j)] = g.param;
}

template <int GROUP, int BITS, bool FB, int QM, bool RK = false>
__global__ void __launch_bounds__(kPipeThreads, 2) k_quantize_tma(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int M = FB ? 1 : kQuantizeSubtilesNF;
    constexpr int NS = FB ? kStagesQuantizeFB : kStagesQuantizeNF;
    const PipeShared p = pipe_shared<NS>(smem);
    griddep_launch_dependents();
    pipe_init<NS>(p);
    const int warp = threadIdx.x >> 5;
    RunWalker<GROUP, M, RK, 0> walker(a);
    if (warp == kConsumerWarps) {
        if ((threadIdx.x & 31) == 0) produce<GROUP, M, NS, RK, 0>(a, p, walker, FB);
        return;
    }
    // with feedback: 8 elements per lane, one pass per tile; without: 32 per
    // lane, one pass over the 4-sub-tile stage
    using LNF = LaneE<GROUP, kQuantizeLaneElemsNF>;
    constexpr int GPW = FB ? Lane<GROUP>::GPW : LNF::GPW;
    constexpr int PASSES = FB ? 1 : M * kTileElems / (kConsumerWarps * 32 * kQuantizeLaneElemsNF);
    static_assert(FB || PASSES * kConsumerWarps * 32 * kQuantizeLaneElemsNF == M * kTileElems, "tile split");
    const int gi = warp * GPW + (FB ? Lane<GROUP>().sub : LNF().sub);
    const bool lead = (threadIdx.x & 31) == 0;
    long long i = 0;
    Tile t;
    for (long long k = blockIdx.x; walker.locate(k, &t, a); k += gridDim.x, ++i) {
        const int s = (int)(i % NS);
        if (!mbar_wait(&p.full[s], (uint32_t)(i / NS) & 1u, a.wait_ns, p.abort)) {
            if (lead) {
                report_timeout(a, p);
                if (FB) bulk_wait_all();   // this warp's stores still in flight
            }
            return;
        }
        uint8_t* stage = p.stages + (size_t)s * kStageBytes;
        if (FB) {
            quantize_tile_group<GROUP, BITS, QM, RK>(a, stage, t, gi, gi < t.count);
            // The warp's groups are GPW consecutive groups of the tile: their
            // updated EMA rows leave the stage in two bulk stores. The slot is
            // released once those stores have read it, one tile later.
            fence_proxy_async_smem();
            __syncwarp();
            if (lead) {
                const int g0 = warp * GPW;
                const int cnt = min(GPW, t.count - g0);
                if (cnt > 0) {
                    const uint32_t bytes = (uint32_t)cnt * GROUP * 4;
                    float* el = state_row_t<RK>(a, t.rank) + (t.j0 + g0) * GROUP;
                    bulk_store(el, stage + kTileElems * 2 + g0 * GROUP * 4, bytes);
                    bulk_store(el + a.S, stage + kTileElems * 6 + g0 * GROUP * 4, bytes);
                }
                bulk_commit();
                bulk_wait_read<1>();
                if (i > 0) mbar_arrive(&p.empty[(i - 1) % NS]);
            }
            __syncwarp();
            continue;
        } else {
#pragma unroll 1
            for (int m = 0; m < PASSES; ++m) {
                const int g = gi + m * kConsumerWarps * GPW;
                quantize_tile_group_nf<GROUP, BITS, QM, RK>(a, stage, t, g, g < t.count);
            }
        }
        __syncwarp();
        if (lead) mbar_arrive(&p.empty[s]);
    }
    if (FB && lead) {
        bulk_wait_read<0>();
        if (i > 0) mbar_arrive(&p.empty[(i - 1) % NS]);
        bulk_wait_all();
    }
    // the partial last group (not a multiple of 16 bytes): direct path
    if (a.tail && blockIdx.x == gridDim.x - 1 && warp == 0) {
        const long long j = a.G - 1;
        for (int r = a.rank_lo; r < a.rank_hi; ++r) {
            const long long lo = (long long)r * a.G / a.P, hi = (long long)(r + 1) * a.G / a.P;
            if (j < lo || j >= hi) quantize_range<GROUP, BITS, QM>(a, r, j, j + 1, 0, 1);
        }
    }
}

// ------------------------------------------------------------ reduce

// One owned group of a tile with feedback (x, e_long, e_short staged): 8
// consecutive elements per lane, like the quantize pass.
constexpr int kReduceRankBatch = 8;   // ranks whose payload loads are issued together


// The payload loads of ranks [r0, r0 + RB) for lane t's 8 elements of group
// j: one code word (two at 8 bits) and the group's parameter word per rank;
// zeros for the owner's own slot, ranks past P and inactive lanes.
template <int GROUP, int BITS, bool RK, int RB>
__device__ __forceinline__ void load_payload8(const Args& a, int o, long long j, int t, bool act, int r0,
                                              uint32_t (&cw)[RB][BITS / 4], uint32_t (&pw)[RB]) {
    constexpr int CB = GROUP * BITS / 8, CW = BITS / 4;
#pragma unroll
    for (int k = 0; k < RB; ++k) {
        const int r = r0 + k;
#pragma unroll
        for (int c = 0; c < CW; ++c) cw[k][c] = 0u;
        pw[k] = 0u;
        if (act && r < a.P && r != o) {
            const size_t slot = a2a_slot_t<RK>(a, r, j);
            const uint8_t* codes = a.a2a_codes + slot * CB;
            if (BITS == 4) {
                cw[k][0] = *reinterpret_cast<const uint32_t*>(codes + 4 * t);
            } else {
                const uint2 v = *reinterpret_cast<const uint2*>(codes + 8 * t);
                cw[k][0] = v.x;
                cw[k][CW - 1] = v.y;
            }
            pw[k] = a.a2a_params[slot];
        }
    }
}

// The payload loads of each batch of RB ranks go out together; the first
// batch's before the staged x and EMAs are read, so that their latency
// overlaps the feedback injection. (With the first batch loaded by the caller
// and passed in, the pass ran 1.042 ms against 0.973 at P = 2 and 1.256
// against 1.22 at P = 4 on 512 MB per rank, the same at P = 8; A/B on one
// box.)
template <int GROUP, int BITS, int QM, bool RK>
__device__ __forceinline__ void reduce_tile_group(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                  bool act) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = kReduceRankBatch;
    constexpr int CW = BITS / 4;   // 32-bit code words per lane (8 codes)
    const LN ln;
    const int o = t.rank;
    const long long j = t.j0 + gi;
    const int e0 = 8 * ln.t;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(st) + gi * GROUP;
    const float* els = reinterpret_cast<const float*>(st + kTileElems * 2) + gi * GROUP;
    const float* ess = reinterpret_cast<const float*>(st + kTileElems * 6) + gi * GROUP;
    float2 xo[4], acc[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) xo[p] = acc[p] = make_float2(0.0f, 0.0f);
    // binary32 sum in rank order 0..P-1: own x' unquantized, others decoded
    for (int r0 = 0; r0 < a.P; r0 += RB) {
        uint32_t cw[RB][CW];
        uint32_t pw[RB];
        load_payload8<GROUP, BITS, RK, RB>(a, o, j, ln.t, act, r0, cw, pw);
        if (r0 == 0 && act) {
            // x' = x + c from the staged x and EMAs
            load_x8c_smem(xs + e0, xo);
            float2 el[4], es[4];
            load_f8_smem(els, e0, e0 + 4, el);
            load_f8_smem(ess, e0, e0 + 4, es);
#pragma unroll
            for (int p = 0; p < 4; ++p) xo[p] = inject2(xo[p], el[p], es[p], a);
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            if (r >= a.P) break;
            float2 term[4];
            if (r == o) {
#pragma unroll
                for (int p = 0; p < 4; ++p) term[p] = xo[p];
            } else {
                const float sk = param_s(pw[k]);
                const float2 s2 = splat(sk);
                const float2 z2 = splat(param_zf<QM>(pw[k], sk));
                float2 q[4];
                unpack_codes8<BITS>(cw[k], q);
#pragma unroll
                for (int p = 0; p < 4; ++p) term[p] = fma2_rn(q[p], s2, z2);
            }
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[p] = (r == 0) ? term[p] : add2_rn(acc[p], term[p]);
        }
    }
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
    if (act) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            lmin = nan_min3(lmin, acc[p].x, acc[p].y);
            lmax = nan_max3(lmax, acc[p].x, acc[p].y);
        }
    }
    uint32_t yb[4];   // bf16 pairs of the result
    if (a.P >= 2) {
        const GridP g = make_grid_p<L, Q, QM>(lmin, lmax);
        raise_flags(a, act && g.bad);
        if (!act) return;
        float2 e[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            e[p] = encode2<QM, Q>(acc[p], g, a);
            yb[p] = bf16x2_rn(fma2_rn(add2_rn(e[p], splat(-kMagic)), g.s, g.z));
        }
        uint8_t* codes = a.g_codes + (size_t)(j - a.g_col_base) * CB;
        const uint2 pk = pack_codes8<BITS>(e);
        if (BITS == 4) *reinterpret_cast<uint32_t*>(codes + 4 * ln.t) = pk.x;
        else *reinterpret_cast<uint2*>(codes + 8 * ln.t) = pk;
        if (ln.t == 0) a.g_params[j - a.g_col_base] = g.param;
        if (a.write_outputs) {
            // phase 4 in the owner's pass: every rank's output gets the decoded
            // requantized sum -- the same bits a decode of the gathered payload
            // gives. Plain stores: with the evict-first hint the pass ran
            // 3.49 ms against 3.45 (A/B on one box)
            const uint4 y4 = make_uint4(yb[0], yb[1], yb[2], yb[3]);
            for (int r = 0; r < a.P; ++r) *reinterpret_cast<uint4*>(a.out[r] + j * GROUP + e0) = y4;
        }
    } else {
        // a single rank sends nothing: its output is its own x'
        raise_flags(a, act && !(lmin >= -65504.0f && lmax <= 65504.0f));
        if (!act) return;
#pragma unroll
        for (int p = 0; p < 4; ++p) yb[p] = bf16x2_rn(acc[p]);
        *reinterpret_cast<uint4*>(a.out[0] + j * GROUP + e0) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
    }
    float2 el[4], es[4], nl[4], ns[4];
    load_f8_smem(els, e0, e0 + 4, el);
    load_f8_smem(ess, e0, e0 + 4, es);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        // rho = acc - float(y): flip the sign bits of the bf16 pair, then widen exactly
        const uint32_t ny = yb[p] ^ 0x80008000u;
        const float2 rho = add2_rn(acc[p], make_float2(__uint_as_float(ny << 16), __uint_as_float(ny & 0xffff0000u)));
        nl[p] = ema2(el[p], rho, a.keep_long, a.a_long, a);
        ns[p] = ema2(es[p], rho, a.keep_short, a.a_short, a);
    }
    float* el_g = state_row_t<RK>(a, o) + j * GROUP + e0;
    store_f8_cs(el_g, nl);
    store_f8_cs(el_g + a.S, ns);
}

// One owned group of a tile with feedback, 16 elements per lane: lane t of
// the group's L = GROUP / 16 lanes holds the 8-element chunks t and t + L
// (each chunk's shared-memory reads by 8 lanes cover one contiguous span).
// Against 8 elements per lane, the per-group work -- range reduction, fp16
// parameters, each incoming payload's parameter word and slot address -- is
// shared by twice the elements; a 2048-element tile is one pass of four warps.
template <int GROUP, int BITS, int QM, bool RK>
__device__ __forceinline__ void reduce_tile_group16(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                    bool act) {
    using LN = Lane16<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = BITS == 4 ? 8 : 4;   // ranks whose payload loads are issued together
    constexpr int CW = BITS / 4;            // 32-bit code words per 8-element chunk
    const LN ln;
    const int o = t.rank;
    const long long j = t.j0 + gi;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(st) + gi * GROUP;
    const float* els = reinterpret_cast<const float*>(st + kTileElems * 2) + gi * GROUP;
    const float* ess = reinterpret_cast<const float*>(st + kTileElems * 6) + gi * GROUP;
    float2 xo[8], acc[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) xo[p] = acc[p] = make_float2(0.0f, 0.0f);
    // binary32 sum in rank order 0..P-1: own x' unquantized, others decoded.
    // The first batch's payload loads go out before the staged x and EMAs
    // are read, so that their latency overlaps the feedback injection.
    for (int r0 = 0; r0 < a.P; r0 += RB) {
        uint32_t cw[RB][2 * CW];
        uint32_t pw[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            pw[k] = 0u;
#pragma unroll
            for (int c = 0; c < 2 * CW; ++c) cw[k][c] = 0u;
            if (act && r < a.P && r != o) {
                const size_t slot = a2a_slot_t<RK>(a, r, j);
                const uint8_t* codes = a.a2a_codes + slot * CB;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (BITS == 4) {
                        cw[k][h] = *reinterpret_cast<const uint32_t*>(codes + 4 * ln.chunk(h));
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2*>(codes + 8 * ln.chunk(h));
                        cw[k][2 * h] = v.x;
                        cw[k][2 * h + 1] = v.y;
                    }
                }
                pw[k] = a.a2a_params[slot];
            }
        }
        if (r0 == 0 && act) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e0 = 8 * ln.chunk(h);
                float2 el[4], es[4];
                load_x8c_smem(xs + e0, &xo[4 * h]);
                load_f8_smem(els, e0, e0 + 4, el);
                load_f8_smem(ess, e0, e0 + 4, es);
#pragma unroll
                for (int p = 0; p < 4; ++p) xo[4 * h + p] = inject2(xo[4 * h + p], el[p], es[p], a);
            }
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            if (r >= a.P) break;
            float2 term[8];
            if (r == o) {
#pragma unroll
                for (int p = 0; p < 8; ++p) term[p] = xo[p];
            } else {
                const float sk = param_s(pw[k]);
                const float2 s2 = splat(sk);
                const float2 z2 = splat(param_zf<QM>(pw[k], sk));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float2 q[4];
                    unpack_codes8<BITS>(&cw[k][h * CW], q);
#pragma unroll
                    for (int p = 0; p < 4; ++p) term[4 * h + p] = fma2_rn(q[p], s2, z2);
                }
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) acc[p] = (r == 0) ? term[p] : add2_rn(acc[p], term[p]);
        }
    }
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
    if (act) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            lmin = nan_min3(lmin, acc[p].x, acc[p].y);
            lmax = nan_max3(lmax, acc[p].x, acc[p].y);
        }
    }
    uint32_t yb[8];   // bf16 pairs of the result
    if (a.P >= 2) {
        const GridP g = make_grid_p<L, Q, QM>(lmin, lmax);
        raise_flags(a, act && g.bad);
        if (!act) return;
        uint8_t* codes = a.g_codes + (size_t)(j - a.g_col_base) * CB;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 e[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                e[p] = encode2<QM, Q>(acc[4 * h + p], g, a);
                yb[4 * h + p] = bf16x2_rn(fma2_rn(add2_rn(e[p], splat(-kMagic)), g.s, g.z));
            }
            const uint2 pk = pack_codes8<BITS>(e);
            if (BITS == 4) *reinterpret_cast<uint32_t*>(codes + 4 * ln.chunk(h)) = pk.x;
            else *reinterpret_cast<uint2*>(codes + 8 * ln.chunk(h)) = pk;
        }
        if (ln.t == 0) a.g_params[j - a.g_col_base] = g.param;
        if (a.write_outputs) {
            // phase 4 in the owner's pass: every rank's output gets the decoded
            // requantized sum -- the same bits a decode of the gathered payload
            // gives (plain stores, as in the 8-element pass)
            for (int r = 0; r < a.P; ++r) {
                uint16_t* y = a.out[r] + j * GROUP;
                *reinterpret_cast<uint4*>(y + 8 * ln.chunk(0)) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
                *reinterpret_cast<uint4*>(y + 8 * ln.chunk(1)) = make_uint4(yb[4], yb[5], yb[6], yb[7]);
            }
        }
    } else {
        // a single rank sends nothing: its output is its own x'
        raise_flags(a, act && !(lmin >= -65504.0f && lmax <= 65504.0f));
        if (!act) return;
#pragma unroll
        for (int p = 0; p < 8; ++p) yb[p] = bf16x2_rn(acc[p]);
        uint16_t* y = a.out[0] + j * GROUP;
        *reinterpret_cast<uint4*>(y + 8 * ln.chunk(0)) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
        *reinterpret_cast<uint4*>(y + 8 * ln.chunk(1)) = make_uint4(yb[4], yb[5], yb[6], yb[7]);
    }
    float* el_g = state_row_t<RK>(a, o) + j * GROUP;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int e0 = 8 * ln.chunk(h);
        float2 el[4], es[4], nl[4], ns[4];
        load_f8_smem(els, e0, e0 + 4, el);
        load_f8_smem(ess, e0, e0 + 4, es);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            // rho = acc - float(y): flip the sign bits of the bf16 pair, then widen exactly
            const uint32_t ny = yb[4 * h + p] ^ 0x80008000u;
            const float2 rho = add2_rn(acc[4 * h + p],
                                       make_float2(__uint_as_float(ny << 16), __uint_as_float(ny & 0xffff0000u)));
            nl[p] = ema2(el[p], rho, a.keep_long, a.a_long, a);
            ns[p] = ema2(es[p], rho, a.keep_short, a.a_short, a);
        }
        store_f8_cs(el_g + e0, nl);
        store_f8_cs(el_g + a.S + e0, ns);
    }
}

// The owner's pass without feedback, 16 elements per lane (chunks t and
// t + L16 of 8 elements): twice the elements per payload load batch and per
// group-level step of the 8-element path, and 16-byte output stores.
template <int GROUP, int BITS, int QM, bool RK>
__device__ __forceinline__ void reduce_tile_group_nf(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                     bool act) {
    using LN = Lane16<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = BITS == 4 ? 8 : 4;   // ranks whose payload loads are issued together
    constexpr int CW = BITS / 4;            // 32-bit code words per 8-element chunk
    const LN ln;
    const int o = t.rank;
    const long long j = t.j0 + gi;
    const uint4* xs = reinterpret_cast<const uint4*>(st + (size_t)gi * GROUP * 2);
    uint4 xw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (act) {
        xw[0] = xs[ln.chunk(0)];
        xw[1] = xs[ln.chunk(1)];
    }
    float2 acc[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) acc[p] = make_float2(0.0f, 0.0f);
    // binary32 sum in rank order 0..P-1: own x unquantized, others decoded
    for (int r0 = 0; r0 < a.P; r0 += RB) {
        uint32_t cw[RB][2 * CW];
        uint32_t pw[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            pw[k] = 0u;
#pragma unroll
            for (int c = 0; c < 2 * CW; ++c) cw[k][c] = 0u;
            if (act && r < a.P && r != o) {
                const size_t slot = a2a_slot_t<RK>(a, r, j);
                const uint8_t* codes = a.a2a_codes + slot * CB;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (BITS == 4) {
                        cw[k][h] = *reinterpret_cast<const uint32_t*>(codes + 4 * ln.chunk(h));
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2*>(codes + 8 * ln.chunk(h));
                        cw[k][2 * h] = v.x;
                        cw[k][2 * h + 1] = v.y;
                    }
                }
                pw[k] = a.a2a_params[slot];
            }
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            if (r >= a.P) break;
            float2 term[8];
            if (r == o) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    term[4 * h] = bf16_pair(xw[h].x);
                    term[4 * h + 1] = bf16_pair(xw[h].y);
                    term[4 * h + 2] = bf16_pair(xw[h].z);
                    term[4 * h + 3] = bf16_pair(xw[h].w);
                }
            } else {
                const float sk = param_s(pw[k]);
                const float2 s2 = splat(sk);
                const float2 z2 = splat(param_zf<QM>(pw[k], sk));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float2 q[4];
                    unpack_codes8<BITS>(&cw[k][h * CW], q);
#pragma unroll
                    for (int p = 0; p < 4; ++p) term[4 * h + p] = fma2_rn(q[p], s2, z2);
                }
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) acc[p] = (r == 0) ? term[p] : add2_rn(acc[p], term[p]);
        }
    }
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
    if (act) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            lmin = nan_min3(lmin, acc[p].x, acc[p].y);
            lmax = nan_max3(lmax, acc[p].x, acc[p].y);
        }
    }
    uint32_t yw[8];   // bf16 pairs of the result
    if (a.P >= 2) {
        const GridP g = make_grid_p<L, Q, QM>(lmin, lmax);
        raise_flags(a, act && g.bad);
        if (!act) return;
        uint8_t* codes = a.g_codes + (size_t)(j - a.g_col_base) * CB;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 e[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) e[p] = encode2<QM, Q>(acc[4 * h + p], g, a);
            const uint2 pk = pack_codes8<BITS>(e);
            if (BITS == 4) *reinterpret_cast<uint32_t*>(codes + 4 * ln.chunk(h)) = pk.x;
            else *reinterpret_cast<uint2*>(codes + 8 * ln.chunk(h)) = pk;
#pragma unroll
            for (int p = 0; p < 4; ++p) yw[4 * h + p] = bf16x2_rn(fma2_rn(add2_rn(e[p], splat(-kMagic)), g.s, g.z));
        }
        if (ln.t == 0) a.g_params[j - a.g_col_base] = g.param;
        if (a.write_outputs) {
            // phase 4 in the owner's pass: every rank's output gets the decoded
            // requantized sum -- the same bits a decode of the gathered payload
            // gives (plain stores, as in the 8-element pass)
            for (int r = 0; r < a.P; ++r) {
                uint16_t* y = a.out[r] + j * GROUP;
                *reinterpret_cast<uint4*>(y + 8 * ln.chunk(0)) = make_uint4(yw[0], yw[1], yw[2], yw[3]);
                *reinterpret_cast<uint4*>(y + 8 * ln.chunk(1)) = make_uint4(yw[4], yw[5], yw[6], yw[7]);
            }
        }
    } else {
        // a single rank sends nothing: its output is its own x
        raise_flags(a, act && !(lmin >= -65504.0f && lmax <= 65504.0f));
        if (!act) return;
#pragma unroll
        for (int p = 0; p < 8; ++p) yw[p] = bf16x2_rn(acc[p]);
        uint16_t* y = a.out[0] + j * GROUP;
        *reinterpret_cast<uint4*>(y + 8 * ln.chunk(0)) = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        *reinterpret_cast<uint4*>(y + 8 * ln.chunk(1)) = make_uint4(yw[4], yw[5], yw[6], yw[7]);
    }
}

// One rank of a multi-GPU call without feedback: 16 consecutive elements per
// lane, so that a received row's codes for them are one 8-byte load (16 bytes
// at 8 bits) and the gather payload's one store (against two 4-byte ones with
// chunks t and t + L: 0.191 -> 0.172 ms on the 1 GB P = 8 message, A/B on one
// box; the simulation's pass, with its P output stores, ran 1.97 -> 2.21 ms
// in this layout and keeps the other). Lanes of a group past the tile's end
// load the tile's last group (every address stays inside the received rows,
// this rank's own unused row included) and store nothing, so the loads need
// no predicate. The own x is read from the staged tile when its turn in the
// rank order comes rather than held in registers through the sum (0.171 ->
// 0.162 ms), and the sum starts from zeros only to keep the register
// allocator from spilling (every element's first term replaces it).
template <int GROUP, int BITS, int QM>
__device__ __forceinline__ void reduce_tile_group_nf_rank(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                          bool act) {
    using LN = Lane16<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = BITS == 4 ? 8 : 4;   // ranks whose payload loads are issued together
    constexpr int CW = BITS / 2;            // 32-bit code words per 16 elements
    const LN ln;
    const int o = t.rank;
    const long long j = t.j0 + gi;
    const long long jl = t.j0 + min(gi, t.count - 1);
    const uint4* xs = reinterpret_cast<const uint4*>(st + (size_t)gi * GROUP * 2) + 2 * ln.t;
    float2 acc[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) acc[p] = make_float2(0.0f, 0.0f);
    // binary32 sum in rank order 0..P-1: own x unquantized, others decoded
    for (int r0 = 0; r0 < a.P; r0 += RB) {
        uint32_t cw[RB][CW];
        uint32_t pw[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const size_t slot = a2a_slot(a, min(r0 + k, a.P - 1), jl);
            const uint8_t* codes = a.a2a_codes + slot * CB + 4 * CW * ln.t;
            if (BITS == 4) {
                const uint2 v = *reinterpret_cast<const uint2*>(codes);
                cw[k][0] = v.x;
                cw[k][1] = v.y;
            } else {
                const uint4 v = *reinterpret_cast<const uint4*>(codes);
                cw[k][0] = v.x;
                cw[k][1] = v.y;
                cw[k][2] = v.z;
                cw[k][3] = v.w;
            }
            pw[k] = a.a2a_params[slot];
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            if (r >= a.P) break;
            float2 term[8];
            if (r == o) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 xh = xs[h];   // read when its turn comes: no registers held through the sum
                    term[4 * h] = bf16_pair(xh.x);
                    term[4 * h + 1] = bf16_pair(xh.y);
                    term[4 * h + 2] = bf16_pair(xh.z);
                    term[4 * h + 3] = bf16_pair(xh.w);
                }
            } else {
                const float sk = param_s(pw[k]);
                const float2 s2 = splat(sk);
                const float2 z2 = splat(param_zf<QM>(pw[k], sk));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float2 q[4];
                    unpack_codes8<BITS>(&cw[k][h * CW / 2], q);
#pragma unroll
                    for (int p = 0; p < 4; ++p) term[4 * h + p] = fma2_rn(q[p], s2, z2);
                }
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) acc[p] = (r == 0) ? term[p] : add2_rn(acc[p], term[p]);
        }
    }
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        lmin = nan_min3(lmin, acc[p].x, acc[p].y);
        lmax = nan_max3(lmax, acc[p].x, acc[p].y);
    }
    if (a.P >= 2) {
        const GridP g = make_grid_p<L, Q, QM>(lmin, lmax);
        raise_flags(a, act && g.bad);
        if (!act) return;
        uint8_t* codes = a.g_codes + (size_t)(j - a.g_col_base) * CB + 4 * CW * ln.t;
        uint2 pk[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 e[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) e[p] = encode2<QM, Q>(acc[4 * h + p], g, a);
            pk[h] = pack_codes8<BITS>(e);
        }
        if (BITS == 4) *reinterpret_cast<uint2*>(codes) = make_uint2(pk[0].x, pk[1].x);
        else *reinterpret_cast<uint4*>(codes) = make_uint4(pk[0].x, pk[0].y, pk[1].x, pk[1].y);
        if (ln.t == 0) a.g_params[j - a.g_col_base] = g.param;
    } else {
        // a single rank sends nothing: its output is its own x
        raise_flags(a, act && !(lmin >= -65504.0f && lmax <= 65504.0f));
        if (!act) return;
        uint32_t yw[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) yw[p] = bf16x2_rn(acc[p]);
        uint4* y = reinterpret_cast<uint4*>(a.out[o] + j * GROUP) + 2 * ln.t;
        y[0] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        y[1] = make_uint4(yw[4], yw[5], yw[6], yw[7]);
    }
}

// Two CTAs of kPipeThreads per SM: 96 registers per thread (each SM
// sub-partition's 16384 registers then hold its share of the 18 warps).
// WIDE: the simulation with feedback and P > kReduceRankBatch.
template <int GROUP, int BITS, bool FB, int QM, bool RK = false, bool WIDE = false>
__global__ void __launch_bounds__(kPipeThreads, 2) k_reduce_tma(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int M = FB ? 1 : kReduceSubtilesNF;
    constexpr int NS = FB ? kStagesReduceFB : kStagesReduceNF;
    // One rank of a multi-GPU call with feedback, and the simulation with
    // feedback at P > kReduceRankBatch: 16 elements per lane, the two halves
    // of the consumer warps taking alternate tiles (each stage is released by
    // one half), so that the per-group work of each incoming payload (its
    // parameter word, its slot address) serves twice the elements. The
    // simulation with feedback at P <= kReduceRankBatch: 8 elements per lane,
    // all consumer warps on every tile (the halves measured 2.6 % slower
    // there; at P = 16 they took the pass from 2.85 to 2.77 ms, 85.6 ->
    // 88.1 % of its roofline on 512 MB per rank, A/B on one box). Without
    // feedback: 16 elements per lane, two passes of all warps over a
    // 4-sub-tile stage.
    constexpr bool HALVES = FB && (RK || WIDE);
    const PipeShared p = pipe_shared<NS>(smem);
    pipe_init<NS>(p, HALVES ? kConsumerWarps / 2 : kConsumerWarps);
    const int warp = threadIdx.x >> 5;
    RunWalker<GROUP, M, RK, 1> walker(a);
    if (warp == kConsumerWarps) {
        // the owned groups' x and EMAs: the quantize pass writes neither, so
        // the producer may stage them while that pass is still running
        if ((threadIdx.x & 31) == 0) produce<GROUP, M, NS, RK, 1, RK ? GROUP * BITS / 8 : 0>(a, p, walker, FB);
        return;
    }
    // the payload, the flag word and the outputs: only once the quantize pass
    // is complete (an output may be the same buffer as an input it reads)
    griddep_wait();
    const bool lead = (threadIdx.x & 31) == 0;
    Tile t;
    if (FB && !HALVES) {
        // The simulation at P <= kReduceRankBatch: 8 elements per lane, the
        // payload loaded once the tile is staged (issuing the first batch
        // before the wait measured 1-2 % slower)
        const int gi = warp * Lane<GROUP>::GPW + Lane<GROUP>().sub;
        long long i = 0;
        for (long long k = blockIdx.x; walker.locate(k, &t, a); k += gridDim.x, ++i) {
            const int s = (int)(i % NS);
            if (!mbar_wait(&p.full[s], (uint32_t)(i / NS) & 1u, a.wait_ns, p.abort)) {
                if (lead) report_timeout(a, p);
                return;
            }
            reduce_tile_group<GROUP, BITS, QM, RK>(a, p.stages + (size_t)s * kStageBytes, t, gi, gi < t.count);
            __syncwarp();
            if (lead) mbar_arrive(&p.empty[s]);
        }
    } else {
        constexpr int GPW = Lane16<GROUP>::GPW;
        constexpr int HALF = kConsumerWarps / 2;
        constexpr int PASSES = FB ? 1 : M * kTileElems / (kConsumerWarps * 32 * 16);
        constexpr int STEP = HALVES ? 2 : 1;
        static_assert(!HALVES || HALF * GPW * GROUP == kTileElems, "a tile is one pass of half the consumer warps");
        const int half = HALVES ? warp / HALF : 0;
        const int gi = (HALVES ? warp % HALF : warp) * GPW + Lane16<GROUP>().sub;
        long long i = half;
        for (long long k = blockIdx.x + half * gridDim.x; walker.locate(k, &t, a); k += STEP * gridDim.x, i += STEP) {
            const int s = (int)(i % NS);
            if (!mbar_wait(&p.full[s], (uint32_t)(i / NS) & 1u, a.wait_ns, p.abort)) {
                if (lead) report_timeout(a, p);
                return;
            }
            const uint8_t* stage = p.stages + (size_t)s * kStageBytes;
            if (FB) {
                reduce_tile_group16<GROUP, BITS, QM, RK>(a, stage, t, gi, gi < t.count);
            } else {
#pragma unroll 1
                for (int m = 0; m < PASSES; ++m) {
                    const int g = gi + m * kConsumerWarps * GPW;
                    if (RK)
                        reduce_tile_group_nf_rank<GROUP, BITS, QM>(a, stage, t, g, g < t.count);
                    else
                        reduce_tile_group_nf<GROUP, BITS, QM, false>(a, stage, t, g, g < t.count);
                }
            }
            __syncwarp();
            if (lead) mbar_arrive(&p.empty[s]);
        }
    }
    if (a.tail && blockIdx.x == gridDim.x - 1 && warp == 0) {
        const long long j = a.G - 1;
        const int o = (int)((j * a.P + a.P - 1) / a.G);
        if (o >= a.rank_lo && o < a.rank_hi) reduce_range<GROUP, BITS, QM>(a, o, j, j + 1, 0, 1);
    }
}

// ------------------------------------------------------------ gather
//
// Every rank receives the same decoded group, so the kernel decodes a tile of
// the gathered payload once into shared memory and sends it to the P outputs
// with P bulk stores (the TMA engine writes; no per-thread store traffic).
// A ring of kGatherBufs tile buffers lets decoding run ahead of the stores.

constexpr int kGatherThreads = 256;
constexpr int kGatherTileElems = kGatherThreads * 8;                 // 2048 elements, 4 KB of bf16
constexpr int kGatherBufs = 4;
constexpr int kGatherSmem = kGatherBufs * kGatherTileElems * 2;     // 16 KB


// eight contiguous decoded elements of a group as bf16 (codes word w: 4-bit in
// w.x, 8-bit in w.x and w.y)
template <int BITS, int QM>
__device__ __forceinline__ uint4 decode8_bf16(uint2 w, uint32_t param) {
    const float s = param_s(param);
    const float2 s2 = splat(s);
    const float2 z2 = splat(param_zf<QM>(param, s));
    float2 q[4];
    const uint32_t cw[2] = {w.x, w.y};
    unpack_codes8<BITS>(cw, q);
    return make_uint4(bf16x2_rn(fma2_rn(q[0], s2, z2)), bf16x2_rn(fma2_rn(q[1], s2, z2)),
                      bf16x2_rn(fma2_rn(q[2], s2, z2)), bf16x2_rn(fma2_rn(q[3], s2, z2)));
}

template <int GROUP, int BITS, int QM>
__global__ void __launch_bounds__(kGatherThreads) k_gather_tma(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int L = GROUP / 8, CB = GROUP * BITS / 8, T = kGatherTileElems / GROUP;
    const long long c1 = a.c1;   // full groups of the column window [c0, c1)
    const long long ntiles = c1 > a.c0 ? (c1 - a.c0 + T - 1) / T : 0;
    const int tid = threadIdx.x;
    const int gi = tid / L, t = tid % L;   // group within the tile, lane within the group
    long long i = 0;
    for (long long k = blockIdx.x; k < ntiles; k += gridDim.x, ++i) {
        const int b = (int)(i % kGatherBufs);
        uint16_t* buf = reinterpret_cast<uint16_t*>(smem + (size_t)b * kGatherTileElems * 2);
        if (i >= kGatherBufs) {
            // the stores that last read this buffer must be done reading it
            if (tid == 0) bulk_wait_read<kGatherBufs - 1>();
            __syncthreads();
        }
        const long long j0 = a.c0 + k * T;
        const int cnt = (int)min((long long)T, c1 - j0);
        if (gi < cnt) {
            const long long j = j0 + gi;
            const size_t gs = g_read_slot(a, j);
            const uint2 w = load_codes8<BITS>(a.g_codes + gs * CB, t);
            *reinterpret_cast<uint4*>(buf + gi * GROUP + 8 * t) = decode8_bf16<BITS, QM>(w, a.g_params[gs]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            const uint32_t bytes = (uint32_t)cnt * GROUP * 2;
            for (int r = a.out_lo; r < a.out_hi; ++r) bulk_store(a.out[r] + j0 * GROUP, buf, bytes);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    // the partial last group (not a multiple of 16 bytes): direct stores
    if (a.tail && blockIdx.x == gridDim.x - 1 && tid < L) {
        const long long j = a.G - 1;
        const size_t gs = g_read_slot(a, j);
        const uint2 w = load_codes8<BITS>(a.g_codes + gs * CB, tid);
        const uint4 v = decode8_bf16<BITS, QM>(w, a.g_params[gs]);
        const uint32_t yb[4] = {v.x, v.y, v.z, v.w};
        const long long e = j * GROUP + 8 * tid;
        for (int r = a.out_lo; r < a.out_hi; ++r) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (e + k < a.n) a.out[r][e + k] = (uint16_t)(yb[k >> 1] >> (16 * (k & 1)));
        }
    }
}

// Phase 4 on one rank of a multi-GPU call: every group of the gathered
// payload (P owner segments, each padded to g_seg_stride groups) decoded into
// this rank's output (a.out[a.out_lo]). With a single output there is no
// tile to share between stores, so each thread decodes E-element chunks
// straight from registers: the loads of U chunks (one code load and the
// parameter word each) are issued together, then each 16 elements of a chunk
// leave in one 32-byte streaming store (16-byte stores when the output is not
// 32-byte aligned). 32-element chunks (one 16-byte code load at 4 bits) ran
// the 1 GB P = 8 decode in 0.233-0.235 ms against 0.239 with 16-element ones
// (A/B on one box).
//
// Work layout: owner o's run is its segment (in a chunked call, the chunk's
// part of it) clipped to the call's full-group window; a run is cut into
// tiles of TG consecutive groups, and the tiles of all runs are numbered in
// owner order. A CTA walks tiles k = blockIdx.x,
// + gridDim.x, ...: per tile the owner, the first group and the first slot in
// the gathered rows are uniform, so per chunk only 32-bit offsets inside the
// tile are computed. The runs' bounds and tile prefix sums are set up once
// per CTA in shared memory (one thread per owner, then a warp scan).
constexpr int kDecodeThreads = 256;
constexpr int kDecodeUnroll = 8;
constexpr bool kDecodePrefetch = true;   // next tile's loads before this tile's decode
constexpr int kDecodeElems = 32;   // elements per chunk (16 or 32); kDecodeUnroll counts 16-element chunks

// E consecutive codes of a group: E * BITS / 32 words (8, 16 or 32 bytes)
template <int E, int BITS>
struct ChunkCodes {
    static constexpr int W = E * BITS / 32;
    uint32_t w[W];
    __device__ __forceinline__ void load(const uint8_t* p) {
        if (W == 2) {
            const uint2 v = *reinterpret_cast<const uint2*>(p);
            w[0] = v.x;
            w[1] = v.y;
        } else {
#pragma unroll
            for (int q = 0; q < W / 4; ++q) {
                const uint4 v = reinterpret_cast<const uint4*>(p)[q];
                w[4 * q] = v.x;
                w[4 * q + 1] = v.y;
                w[4 * q + 2] = v.z;
                w[4 * q + 3] = v.w;
            }
        }
    }
    // the words of 8-element part k (one at 4 bits, two at 8)
    __device__ __forceinline__ uint2 part(int k) const {
        return BITS == 4 ? make_uint2(w[k], 0u) : make_uint2(w[2 * k], w[2 * k + 1]);
    }
};

template <int GROUP, int BITS, int QM>
__global__ void __launch_bounds__(kDecodeThreads) k_decode_rank(const Args a) {
    constexpr int E = kDecodeElems, L = GROUP / E, CB = GROUP * BITS / 8, U = kDecodeUnroll * 16 / E;
    constexpr int CHUNK_BYTES = E * BITS / 8;
    constexpr int TG = U * kDecodeThreads / L;   // groups per tile
    static_assert((E == 16 || E == 32) && GROUP % E == 0, "16- or 32-element chunks");
    using Codes = ChunkCodes<E, BITS>;
    static_assert(ECHO_MAX_RANKS <= 64, "one warp scans the owners' tile counts");
    __shared__ long long run_b[ECHO_MAX_RANKS], run_e[ECHO_MAX_RANKS], run_slot[ECHO_MAX_RANKS];
    __shared__ long long tile_pre[ECHO_MAX_RANKS + 1];
    const int tid = threadIdx.x;
    if (tid < a.P) {
        const long long sb = (long long)tid * a.G / a.P;
        long long pb, pe;
        segment_part(a, tid, &pb, &pe);   // the segment, or its part for this chunk
        const long long b = max(pb, a.c0), e = max(b, min(pe, a.c1));
        run_b[tid] = b;
        run_e[tid] = e;
        run_slot[tid] = (long long)tid * a.g_seg_stride + (b - sb);
        tile_pre[tid + 1] = (e - b + TG - 1) / TG;   // this owner's tile count, summed below
    }
    __syncthreads();
    if (tid < 32) {   // inclusive scan of the tile counts: lane l holds owners 2l and 2l + 1
        const int o0 = 2 * tid, o1 = 2 * tid + 1;
        const long long c0 = o0 < a.P ? tile_pre[o0 + 1] : 0, c1 = o1 < a.P ? tile_pre[o1 + 1] : 0;
        long long incl = c0 + c1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long v = __shfl_up_sync(kFull, incl, d);
            if (tid >= d) incl += v;
        }
        if (o0 < a.P) tile_pre[o0 + 1] = incl - c1;
        if (o1 < a.P) tile_pre[o1 + 1] = incl;
        if (tid == 0) tile_pre[0] = 0;
    }
    __syncthreads();
    const long long ntiles = tile_pre[a.P];
    // one output (this rank's); 32-byte stores when it is 32-byte aligned
    uint16_t* const out = a.out[a.out_lo];
    const bool v8 = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
    int o = 0;
    // tile k: chunk lc of it covers group lc / L, part lc % L, so its codes
    // start lc * CHUNK_BYTES after the tile's first group's and its output
    // lc * E elements after the tile's first element
    struct TileRef {
        int nchunks;
        const uint8_t* codes;
        const uint32_t* params;
        uint16_t* y;
    };
    auto locate = [&](long long k, TileRef& r) {
        while (k >= tile_pre[o + 1]) ++o;
        const long long off = (k - tile_pre[o]) * TG;
        const long long j0 = run_b[o] + off;
        r.nchunks = (int)min((long long)TG, run_e[o] - j0) * L;
        r.codes = a.g_codes + (size_t)(run_slot[o] + off) * CB;
        r.params = a.g_params + (run_slot[o] + off);
        r.y = out + j0 * GROUP;
    };
    auto load = [&](const TileRef& r, Codes (&w)[U], uint32_t (&pw)[U]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int lc = u * kDecodeThreads + tid;
            if (lc < r.nchunks) {
                w[u].load(r.codes + lc * CHUNK_BYTES);
                pw[u] = r.params[lc / L];
            }
        }
    };
    auto decode_store = [&](const TileRef& r, const Codes (&w)[U], const uint32_t (&pw)[U]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int lc = u * kDecodeThreads + tid;
#pragma unroll
            for (int m = 0; m < E / 16; ++m) {
                if (lc >= r.nchunks) break;
                const uint4 y0 = decode8_bf16<BITS, QM>(w[u].part(2 * m), pw[u]);
                const uint4 y1 = decode8_bf16<BITS, QM>(w[u].part(2 * m + 1), pw[u]);
                uint16_t* dst = r.y + lc * E + 16 * m;
                if (v8) {
                    store_v8_cs(dst, y0, y1);
                } else {
                    __stcs(reinterpret_cast<uint4*>(dst), y0);
                    __stcs(reinterpret_cast<uint4*>(dst + 8), y1);
                }
            }
        }
    };
    if (kDecodePrefetch) {
        // the next tile's loads are issued before this tile is decoded
        long long k = blockIdx.x;
        TileRef cur = {0, nullptr, nullptr, nullptr};
        Codes w[U];
        uint32_t pw[U];
        if (k < ntiles) {
            locate(k, cur);
            load(cur, w, pw);
        }
        while (k < ntiles) {
            const long long kn = k + gridDim.x;
            TileRef nxt = {0, nullptr, nullptr, nullptr};
            Codes wn[U];
            uint32_t pwn[U];
            if (kn < ntiles) {
                locate(kn, nxt);
                load(nxt, wn, pwn);
            }
            decode_store(cur, w, pw);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                w[u] = wn[u];
                pw[u] = pwn[u];
            }
            cur = nxt;
            k = kn;
        }
    } else {
        for (long long k = blockIdx.x; k < ntiles; k += gridDim.x) {
            TileRef cur;
            locate(k, cur);
            Codes w[U];
            uint32_t pw[U];
            load(cur, w, pw);
            decode_store(cur, w, pw);
        }
    }
    // the partial last group (not a multiple of 16 bytes): guarded stores
    if (a.tail && blockIdx.x == gridDim.x - 1 && threadIdx.x < GROUP / 8) {
        const long long j = a.G - 1;
        const size_t gs = g_read_slot(a, j);
        const uint2 w = load_codes8<BITS>(a.g_codes + gs * CB, threadIdx.x);
        const uint4 v = decode8_bf16<BITS, QM>(w, a.g_params[gs]);
        const uint32_t yb[4] = {v.x, v.y, v.z, v.w};
        const long long e = j * GROUP + 8 * threadIdx.x;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (e + k < a.n) out[e + k] = (uint16_t)(yb[k >> 1] >> (16 * (k & 1)));
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
