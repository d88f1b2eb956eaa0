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
//   k_background_traffic  competing HBM traffic: a bulk (TMA) copy that runs
//                         for a duty cycle of every period and sleeps for the
//                         rest, for a fixed wall-clock time, on its own
//                         stream.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "echo_pipeline.cuh"

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

// Competing HBM traffic: one warp per CTA, one CTA per SM; its lane 0
// copies 16 KB chunks of src to dst through a 2-slot shared-memory ring with
// bulk copies (the TMA engine: loads complete on an mbarrier, stores are
// bulk-async groups), so a few registers and 32 KB of shared memory per SM
// keep 32 KB in flight per SM and the kernel fits beside the all-reduce's
// own CTAs. The copy runs during the first on_ns of every period_ns and
// pauses (ring drained, thread asleep) for the rest, until duration_ns have
// passed since the CTA started -- a fixed wall-clock bound: the kernel ends
// by itself whatever else runs. Chunk c of the CTA is global chunk
// blockIdx.x + c * gridDim.x, wrapping around src. Bytes read and written
// are added to *moved (when not null).
constexpr int kBgChunk = 16384;
constexpr int kBgSlots = 2;
constexpr int kBgSmem = kBgChunk * kBgSlots;
constexpr unsigned long long kBgWaitNs = 1000ull * 1000ull * 1000ull;   // 1 s, never reached by a landing load

__global__ void __launch_bounds__(32) k_background_traffic(const uint8_t* src, uint8_t* dst, long long nchunks,
                                                           unsigned long long on_ns, unsigned long long period_ns,
                                                           unsigned long long duration_ns,
                                                           unsigned long long* moved) {
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t bar[kBgSlots];
    if (threadIdx.x != 0) return;
    for (int k = 0; k < kBgSlots; ++k) mbar_init(&bar[k], 1);
    mbar_fence_init();
    const unsigned long long t0 = global_ns();
    unsigned long long copied = 0;
    long long c = blockIdx.x % nchunks;
    uint32_t uses[kBgSlots] = {0u, 0u};   // completed phases of each slot's barrier
    bool failed = false;
    while (!failed) {
        const unsigned long long t = global_ns() - t0;
        if (t >= duration_ns) break;
        const unsigned long long phase = t % period_ns;
        if (phase >= on_ns) {
            const unsigned long long rest = period_ns - phase;
            __nanosleep((unsigned)(rest < 20000ull ? rest : 20000ull));
            continue;
        }
        // a burst of two chunks per slot (128 KB per CTA), then the time is
        // read again
        for (int b = 0; b < 2 && !failed; ++b) {
            long long cc[kBgSlots];
            for (int k = 0; k < kBgSlots; ++k) {
                cc[k] = c;
                mbar_arrive_expect_tx(&bar[k], kBgChunk);
                bulk_load(ring + k * kBgChunk, src + (size_t)c * kBgChunk, kBgChunk, &bar[k]);
                c += gridDim.x;
                if (c >= nchunks) c %= nchunks;
            }
            for (int k = 0; k < kBgSlots; ++k) {
                // the load lands whatever else runs; the limit only guards the
                // wait. On expiry the remaining loads are still waited for
                // (bounded again) before the thread leaves.
                if (!mbar_wait(&bar[k], uses[k] & 1u, kBgWaitNs, nullptr)) {
                    failed = true;
                    for (int q = k; q < kBgSlots; ++q) mbar_wait(&bar[q], uses[q] & 1u, kBgWaitNs, nullptr);
                    break;
                }
                ++uses[k];
                bulk_store(dst + (size_t)cc[k] * kBgChunk, ring + k * kBgChunk, kBgChunk);
                bulk_commit();
                copied += 2ull * kBgChunk;
            }
            bulk_wait_read<0>();   // the slots may be loaded again
        }
    }
    bulk_wait_all();
    if (moved != nullptr) atomicAdd(moved, copied);
}

}  // namespace echo_dev
