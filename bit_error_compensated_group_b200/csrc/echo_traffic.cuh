// echo_traffic.cuh -- the two kernels of the background-traffic study.
//
// The Echo abstract and the explainer's results section ("実測性能と精度")
// report that Echo's advantage over a 16-bit all-reduce grows when other
// traffic competes for the links. On one GPU the shared resource of the
// simulated transport is HBM, so the study runs:
//
//   k_bf16_allreduce_sim  the 16-bit baseline, simulated like Echo over P
//                         virtual ranks: every rank's output is the bf16
//                         rounding of the binary32 sum of the P bf16 inputs
//                         in rank order (no quantization, no state);
//   k_background_traffic  competing HBM traffic: a copy that runs for a duty
//                         cycle of every period and sleeps for the rest, for
//                         a fixed wall-clock time, on its own stream.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace echo_dev {

constexpr int kBf16Threads = 256;
constexpr int kBf16RankBatch = 8;   // ranks whose loads are issued together

// Eight elements per thread per step: one 16-byte load per rank (issued
// kBf16RankBatch ranks at a time), the rank-ordered binary32 sum, one bf16
// rounding, one 16-byte store per rank. `tail_from`: elements from there on
// (fewer than eight) take the scalar path of the last thread.
__global__ void __launch_bounds__(kBf16Threads) k_bf16_allreduce_sim(const Args a) {
    const long long n8 = a.n / 8;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < n8; v += stride) {
        float acc[8];
        for (int r0 = 0; r0 < a.P; r0 += kBf16RankBatch) {
            uint4 w[kBf16RankBatch];
#pragma unroll
            for (int k = 0; k < kBf16RankBatch; ++k)
                if (r0 + k < a.P) w[k] = __ldcs(reinterpret_cast<const uint4*>(a.in[r0 + k]) + v);
#pragma unroll
            for (int k = 0; k < kBf16RankBatch; ++k) {
                if (r0 + k >= a.P) break;
                const uint32_t u[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float lo = bf16_lo(u[q]), hi = bf16_hi(u[q]);
                    if (r0 + k == 0) {
                        acc[2 * q] = lo;
                        acc[2 * q + 1] = hi;
                    } else {
                        acc[2 * q] = __fadd_rn(acc[2 * q], lo);
                        acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], hi);
                    }
                }
            }
        }
        uint4 y;
        y.x = f2bf16(acc[0]) | (f2bf16(acc[1]) << 16);
        y.y = f2bf16(acc[2]) | (f2bf16(acc[3]) << 16);
        y.z = f2bf16(acc[4]) | (f2bf16(acc[5]) << 16);
        y.w = f2bf16(acc[6]) | (f2bf16(acc[7]) << 16);
        for (int r = 0; r < a.P; ++r) __stcs(reinterpret_cast<uint4*>(a.out[r]) + v, y);
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
        for (long long e = n8 * 8; e < a.n; ++e) {
            float acc = 0.0f;
            for (int r = 0; r < a.P; ++r) {
                const float v = __uint_as_float((uint32_t)a.in[r][e] << 16);
                acc = r == 0 ? v : __fadd_rn(acc, v);
            }
            const uint16_t y = (uint16_t)f2bf16(acc);
            for (int r = 0; r < a.P; ++r) a.out[r][e] = y;
        }
    }
}

__device__ __forceinline__ unsigned long long traffic_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Competing HBM traffic. Every thread walks the n16 16-byte words of src
// with the grid stride (wrapping around), copying them to dst during the
// first on_ns of every period_ns and sleeping for the rest, until
// duration_ns have passed since the CTA started (a fixed wall-clock bound:
// the kernel ends by itself whatever else runs). The bytes copied are added
// to *moved (when not null), one atomic per warp.
__global__ void __launch_bounds__(256) k_background_traffic(const uint4* src, uint4* dst, long long n16,
                                                            unsigned long long on_ns, unsigned long long period_ns,
                                                            unsigned long long duration_ns,
                                                            unsigned long long* moved) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) % n16;
    const unsigned long long t0 = traffic_ns();
    unsigned long long copied = 0;
    while (true) {
        const unsigned long long t = traffic_ns() - t0;
        if (t >= duration_ns) break;
        const unsigned long long phase = t % period_ns;
        if (phase < on_ns) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                __stcs(dst + i, __ldcs(src + i));
                i += stride;
                if (i >= n16) i -= n16 * (i / n16);
            }
            copied += 8 * 16;
        } else {
            const unsigned long long rest = period_ns - phase;
            __nanosleep((unsigned)(rest < 20000ull ? rest : 20000ull));
        }
    }
    if (moved != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) copied += __shfl_xor_sync(0xffffffffu, copied, o);
        if ((threadIdx.x & 31) == 0) atomicAdd(moved, 2 * copied);   // read + written
    }
}

}  // namespace echo_dev
