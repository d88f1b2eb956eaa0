// echo_api.cu -- the C ABI declared in include/echo.h: argument checks,
// workspace layout and kernel launches. The library never allocates device
// memory; all work goes on the caller's stream.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>

#include "echo.h"
#include "echo_kernels.cuh"
#include "echo_pipeline.cuh"
#include "echo_traffic.cuh"

struct echo_state {
    int64_t n;
    int P;
    int group;
    int max_bits;
    int64_t G;
    int64_t S;
    float* state;          // nullptr: no feedback
    uint8_t* workspace;
    int device;
    int sm_count;
    int quantizer;         // ECHO_QUANT_*; ECHO_QUANT_DIRECTED unless set
    // echo_allreduce_sim_host: ordering events between the caller's stream and
    // the two copy streams, created on first use, destroyed by echo_free
    cudaEvent_t ev[3];
    bool have_events;
    int rank;              // -1: the single-GPU simulation; else this rank of a multi-GPU call
    uint64_t wait_ns;      // limit of the kernels' bounded waits (echo_set_wait_limit)
};

namespace {

constexpr uint64_t kAlign = 256;
// Launch configurations are cached per device (a process may drive several
// GPUs; the shared-memory opt-in of a kernel is made on each device).
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxN = int64_t(1) << 40;
// bounded device-side waits: default limit and the range echo_set_wait_limit accepts
constexpr uint64_t kDefaultWaitNs = 1000ull * 1000ull * 1000ull;   // 1 s
constexpr uint32_t kMinWaitUs = 1000u, kMaxWaitUs = 60u * 1000u * 1000u;

uint64_t align_up(uint64_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool valid_group(int g) { return g == 32 || g == 64 || g == 128 || g == 256; }
bool valid_bits(int b) { return b == 4 || b == 8; }
bool valid_sizes(int64_t n, int P, int group) {
    return n >= 1 && n < kMaxN && P >= 1 && P <= ECHO_MAX_RANKS && valid_group(group);
}
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool in_unit(float v) { return v >= 0.0f && v <= 1.0f; }   // NaN fails

bool layout(int64_t n, int P, int group, int max_bits, int bits, echo_layout* L) {
    if (!valid_sizes(n, P, group) || !valid_bits(max_bits) || !valid_bits(bits) || bits > max_bits) return false;
    const uint64_t G = (uint64_t)((n + group - 1) / group);
    const uint64_t cb_max = (uint64_t)group * (uint64_t)max_bits / 8;
    L->groups = (int64_t)G;
    L->state_stride = (int64_t)(G * (uint64_t)group);
    L->code_bytes = (uint64_t)group * (uint64_t)bits / 8;
    uint64_t off = 0;
    L->flags_offset = off;
    off += kAlign;
    L->a2a_codes_offset = off;
    off = align_up(off + (uint64_t)P * G * cb_max);
    L->a2a_params_offset = off;
    off = align_up(off + (uint64_t)P * G * 4);
    L->gather_codes_offset = off;
    off = align_up(off + G * cb_max);
    L->gather_params_offset = off;
    off = align_up(off + G * 4);
    L->workspace_bytes = off;
    L->state_bytes = (uint64_t)P * 2 * G * (uint64_t)group * sizeof(float);
    return true;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? ECHO_OK : ECHO_ECUDA; }

template <typename K>
int grid_for(K kernel, const echo_state* st, int threads = echo_dev::kThreads, int smem = 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess ||
        per_sm < 1) {
        per_sm = 1;
    }
    return st->sm_count * per_sm;
}

// Pipelined kernels: opt in to their dynamic shared memory once.
template <typename K>
int pipe_grid(K kernel, const echo_state* st, int smem) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
        return 0;
    }
    return grid_for(kernel, st, echo_dev::kPipeThreads, smem);
}

enum class Stage { Quantize, Reduce, Gather };


// An upper bound on the tiles a pipelined launch walks: the runs (2 per rank
// for quantize, 1 per owner for reduce) cut into tiles of `tile_groups`.
int64_t tile_bound(Stage stage, const echo_dev::Args& a, int tile_groups) {
    int64_t cols = a.c1 - a.c0;   // the call's group-column window
    if (a.chunk_k > 0) cols = cols / a.chunk_k + a.P;   // every owner's part of one chunk
    const int64_t groups = stage == Stage::Quantize ? (int64_t)(a.P - 1) * cols : cols;
    const int64_t runs = stage == Stage::Quantize ? (a.chunk_k > 0 ? (int64_t)a.P * a.P : 2 * (int64_t)a.P) : a.P;
    return groups / tile_groups + runs + 1;
}

// One pipelined launch; `grids` caches, per device, the grid (and the
// shared-memory opt-in) of this kernel instantiation. A persistent launch
// never needs more CTAs than tiles: small messages then start only the CTAs
// that have work. `pdl`: launch as a programmatic dependent of the kernel
// before it on the stream (the owners' pass right after this call's quantize
// pass).
template <typename K>
int launch_pipe(K kernel, int* grids, int64_t max_tiles, const echo_dev::Args& a, const echo_state* st,
                cudaStream_t s, int smem, bool pdl = false) {
    int& grid = grids[st->device];
    if (grid == 0) grid = pipe_grid(kernel, st, smem);
    if (grid == 0) return ECHO_ECUDA;
    const int g = (int)(max_tiles < (int64_t)grid ? max_tiles : (int64_t)grid);
    if (!pdl) {
        kernel<<<g, echo_dev::kPipeThreads, smem, s>>>(a);
        return ECHO_OK;
    }
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g);
    cfg.blockDim = dim3(echo_dev::kPipeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a) == cudaSuccess ? ECHO_OK : ECHO_ECUDA;
}

template <int GROUP, int BITS, int QM>
int launch_stage(Stage stage, const echo_dev::Args& a, const echo_state* st, cudaStream_t s, bool pdl) {
    int rc = ECHO_OK;
    // tiles of kTileElems elements with feedback; without, the sub-tile
    // counts of the kernels' RunWalkers (kQuantizeSubtilesNF, kReduceSubtilesNF)
    const int subtiles = a.state ? 1
                         : stage == Stage::Quantize ? echo_dev::kQuantizeSubtilesNF
                                                    : echo_dev::kReduceSubtilesNF;
    const int64_t tiles = tile_bound(stage, a, subtiles * echo_dev::kTileElems / GROUP);
    switch (stage) {
        case Stage::Quantize:
            if (st->rank >= 0 && a.state) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_quantize_tma<GROUP, BITS, true, QM, true>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesQuantizeFB));
            } else if (st->rank >= 0) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_quantize_tma<GROUP, BITS, false, QM, true>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesQuantizeNF));
            } else if (a.state) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_quantize_tma<GROUP, BITS, true, QM>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesQuantizeFB));
            } else {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_quantize_tma<GROUP, BITS, false, QM>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesQuantizeNF));
            }
            break;
        case Stage::Reduce:
            // one rank of a multi-GPU call reads its received rows: the
            // instantiation with the general slot addressing
            if (st->rank >= 0 && a.state) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_reduce_tma<GROUP, BITS, true, QM, true>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesReduceFB), pdl);
            } else if (st->rank >= 0) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_reduce_tma<GROUP, BITS, false, QM, true>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesReduceNF), pdl);
            } else if (a.state && a.P > echo_dev::kReduceRankBatch) {
                // more incoming payloads than one load batch: 16 elements per
                // lane, the consumer halves taking alternate tiles
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_reduce_tma<GROUP, BITS, true, QM, false, true>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesReduceFB), pdl);
            } else if (a.state) {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_reduce_tma<GROUP, BITS, true, QM>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesReduceFB), pdl);
            } else {
                static int grid[kMaxDevices];
                rc = launch_pipe(echo_dev::k_reduce_tma<GROUP, BITS, false, QM>, grid, tiles, a, st, s,
                                 echo_dev::pipe_smem(echo_dev::kStagesReduceNF), pdl);
            }
            break;
        case Stage::Gather: {
            if (st->rank >= 0) {   // one rank's output: the register-path decoder
                auto k = echo_dev::k_decode_rank<GROUP, BITS, QM>;
                static int grid[kMaxDevices];
                int& g = grid[st->device];
                if (g == 0) g = grid_for(k, st, echo_dev::kDecodeThreads, 0);
                k<<<g, echo_dev::kDecodeThreads, 0, s>>>(a);
                break;
            }
            auto k = echo_dev::k_gather_tma<GROUP, BITS, QM>;
            static int grid[kMaxDevices];
            int& g = grid[st->device];
            if (g == 0) g = grid_for(k, st, echo_dev::kGatherThreads, echo_dev::kGatherSmem);
            k<<<g, echo_dev::kGatherThreads, echo_dev::kGatherSmem, s>>>(a);
            break;
        }
    }
    if (rc != ECHO_OK) return rc;
    return cuda_status(cudaGetLastError());
}

template <int GROUP>
int launch_bits(Stage stage, int bits, const echo_dev::Args& a, const echo_state* st, cudaStream_t s, bool pdl) {
    switch (st->quantizer) {
        case ECHO_QUANT_DIRECTED:
            return bits == 4 ? launch_stage<GROUP, 4, echo_dev::kQuantDirected>(stage, a, st, s, pdl)
                             : launch_stage<GROUP, 8, echo_dev::kQuantDirected>(stage, a, st, s, pdl);
        case ECHO_QUANT_NEAREST:
            return bits == 4 ? launch_stage<GROUP, 4, echo_dev::kQuantNearest>(stage, a, st, s, pdl)
                             : launch_stage<GROUP, 8, echo_dev::kQuantNearest>(stage, a, st, s, pdl);
        case ECHO_QUANT_INT_ZERO:
            return bits == 4 ? launch_stage<GROUP, 4, echo_dev::kQuantIntZero>(stage, a, st, s, pdl)
                             : launch_stage<GROUP, 8, echo_dev::kQuantIntZero>(stage, a, st, s, pdl);
    }
    return ECHO_EINVAL;
}

// `pdl` (owners' pass only): this launch directly follows the same call's
// quantize launch on the stream and may overlap its tail.
// echo_inject_launch_failure: while set, launches report ECHO_ECUDA instead
std::atomic<int> g_fail_launches{0};

int launch(Stage stage, int bits, const echo_dev::Args& a, const echo_state* st, cudaStream_t s, bool pdl = false) {
    if (g_fail_launches.load(std::memory_order_relaxed)) return ECHO_ECUDA;
    switch (st->group) {
        case 32: return launch_bits<32>(stage, bits, a, st, s, pdl);
        case 64: return launch_bits<64>(stage, bits, a, st, s, pdl);
        case 128: return launch_bits<128>(stage, bits, a, st, s, pdl);
        case 256: return launch_bits<256>(stage, bits, a, st, s, pdl);
    }
    return ECHO_EINVAL;
}

// The call's group columns [c0, c1) as the kernels take them: the full
// groups of the window, and whether it holds the partial last group.
void set_window(echo_dev::Args* a, const echo_state* st, int64_t c0, int64_t c1) {
    const int64_t full = st->n / st->group;
    a->c0 = c0;
    a->c1 = c1 < full ? c1 : full;
    a->tail = (full < st->G && c1 == st->G) ? 1 : 0;
}

bool valid_feedback(float eta, float aL, float aS, float w) {
    return std::isfinite(eta) && in_unit(aL) && in_unit(aS) && in_unit(w);
}

// Fill the kernel arguments; false when a pointer is missing or misaligned.
bool make_args(const echo_state* st, int bits, const void* const* inputs, void* const* outputs,
               float eta, float aL, float aS, float w, echo_dev::Args* a) {
    std::memset(a, 0, sizeof(*a));
    echo_layout L;
    if (!layout(st->n, st->P, st->group, st->max_bits, bits, &L)) return false;
    for (int r = 0; r < st->P; ++r) {
        if (inputs) {
            if (!inputs[r] || !aligned(inputs[r], 16)) return false;
            a->in[r] = static_cast<const uint16_t*>(inputs[r]);
        }
        if (outputs) {
            if (!outputs[r] || !aligned(outputs[r], 16)) return false;
            a->out[r] = static_cast<uint16_t*>(outputs[r]);
        }
    }
    a->state = st->state;
    a->a2a_codes = st->workspace + L.a2a_codes_offset;
    a->a2a_params = reinterpret_cast<uint32_t*>(st->workspace + L.a2a_params_offset);
    a->g_codes = st->workspace + L.gather_codes_offset;
    a->g_params = reinterpret_cast<uint32_t*>(st->workspace + L.gather_params_offset);
    a->flags = reinterpret_cast<uint32_t*>(st->workspace + L.flags_offset);
    a->n = st->n;
    a->G = st->G;
    set_window(a, st, 0, st->G);
    // every rank, in the simulation's layouts
    a->rank_lo = 0;
    a->rank_hi = st->P;
    a->a2a_stride = st->G;
    a->out_lo = 0;
    a->out_hi = st->P;
    a->S = st->S;
    a->P = st->P;
    a->eta = eta;
    a->w = w;
    a->one_minus_w = 1.0f - w;
    a->a_long = aL;
    a->keep_long = 1.0f - aL;
    a->a_short = aS;
    a->keep_short = 1.0f - aS;
    a->one = 1.0f;
    a->wait_ns = st->wait_ns;
    return true;
}

// Layout of one rank's workspace in a multi-GPU call (see echo_rank_layout).
bool rank_layout(int64_t n, int P, int rank, int group, int max_bits, int bits, echo_rank_layout* L) {
    if (!valid_sizes(n, P, group) || !valid_bits(max_bits) || !valid_bits(bits) || bits > max_bits) return false;
    if (rank < 0 || rank >= P) return false;
    const int64_t G = (n + group - 1) / group;
    const uint64_t cb = (uint64_t)group * (uint64_t)bits / 8, cb_max = (uint64_t)group * (uint64_t)max_bits / 8;
    int64_t seg_max = 0;
    for (int s = 0; s < P; ++s) {
        const int64_t len = (int64_t)(s + 1) * G / P - (int64_t)s * G / P;
        if (len > seg_max) seg_max = len;
    }
    L->groups = G;
    L->seg_begin = (int64_t)rank * G / P;
    L->seg_groups = (int64_t)(rank + 1) * G / P - L->seg_begin;
    L->seg_max = seg_max;
    L->code_bytes = cb;
    const uint64_t Pu = (uint64_t)P, Gu = (uint64_t)G, seg = (uint64_t)L->seg_groups, sm = (uint64_t)seg_max;
    uint64_t off = 0;
    L->flags_offset = off;
    off += kAlign;
    L->send_codes_offset = off;
    off = align_up(off + Gu * cb_max);
    L->send_params_offset = off;
    off = align_up(off + Gu * 4);
    L->recv_codes_offset = off;
    off = align_up(off + Pu * seg * cb_max);
    L->recv_params_offset = off;
    off = align_up(off + Pu * seg * 4);
    L->gsend_codes_offset = off;
    off = align_up(off + sm * cb_max);
    L->gsend_params_offset = off;
    off = align_up(off + sm * 4);
    L->grecv_codes_offset = off;
    off = align_up(off + Pu * sm * cb_max);
    L->grecv_params_offset = off;
    off = align_up(off + Pu * sm * 4);
    L->workspace_bytes = off;
    L->state_bytes = 2 * Gu * (uint64_t)group * sizeof(float);
    return true;
}

// Kernel arguments of one rank's phase. `x` / `out`: this rank's input and
// output (either may be null where the phase does not use it).
enum class RankPhase { Quantize, Reduce, Decode };

bool make_rank_args(const echo_state* st, int bits, RankPhase phase, const void* x, void* out, float eta, float aL,
                    float aS, float w, echo_dev::Args* a) {
    std::memset(a, 0, sizeof(*a));
    echo_rank_layout L;
    if (!rank_layout(st->n, st->P, st->rank, st->group, st->max_bits, bits, &L)) return false;
    const int r = st->rank;
    if (x) {
        if (!aligned(x, 16)) return false;
        a->in[r] = static_cast<const uint16_t*>(x);
    }
    if (out) {
        if (!aligned(out, 16)) return false;
        a->out[r] = static_cast<uint16_t*>(out);
    }
    uint8_t* ws = st->workspace;
    a->state = st->state;
    a->state_rank_base = r;
    a->flags = reinterpret_cast<uint32_t*>(ws + L.flags_offset);
    a->n = st->n;
    a->G = st->G;
    a->S = st->S;
    a->P = st->P;
    set_window(a, st, 0, st->G);
    a->rank_lo = r;
    a->rank_hi = r + 1;
    a->out_lo = r;
    a->out_hi = r + 1;
    switch (phase) {
        case RankPhase::Quantize:   // this rank's row of slots [r][j], all j
            a->a2a_codes = ws + L.send_codes_offset;
            a->a2a_params = reinterpret_cast<uint32_t*>(ws + L.send_params_offset);
            a->a2a_rank_base = r;
            a->a2a_stride = st->G;
            break;
        case RankPhase::Reduce:     // slots [r'][j] of this rank's segment, received from every r'
            a->a2a_codes = ws + L.recv_codes_offset;
            a->a2a_params = reinterpret_cast<uint32_t*>(ws + L.recv_params_offset);
            a->a2a_stride = L.seg_groups;
            a->a2a_col_base = L.seg_begin;
            a->g_codes = ws + L.gsend_codes_offset;
            a->g_params = reinterpret_cast<uint32_t*>(ws + L.gsend_params_offset);
            a->g_col_base = L.seg_begin;
            a->write_outputs = st->P == 1;   // a single rank's output comes from this pass
            break;
        case RankPhase::Decode:     // every owner's segment, gathered and padded to seg_max
            a->g_codes = ws + L.grecv_codes_offset;
            a->g_params = reinterpret_cast<uint32_t*>(ws + L.grecv_params_offset);
            a->g_seg_stride = L.seg_max;
            break;
    }
    a->eta = eta;
    a->w = w;
    a->one_minus_w = 1.0f - w;
    a->a_long = aL;
    a->keep_long = 1.0f - aL;
    a->a_short = aS;
    a->keep_short = 1.0f - aS;
    a->one = 1.0f;
    a->wait_ns = st->wait_ns;
    return true;
}

// One chunk of a chunked rank call: chunk `chunk` of `chunks` of every
// owner's segment; the partial last group (the last group of the last
// owner's segment) belongs to the last chunk.
bool set_chunk(echo_dev::Args* a, const echo_state* st, int chunk, int chunks) {
    if (chunks < 1 || chunks > ECHO_MAX_CHUNKS || chunk < 0 || chunk >= chunks) return false;
    if (chunks == 1) return true;   // the whole call
    a->chunk_i = chunk;
    a->chunk_k = chunks;
    const int64_t full = st->n / st->group;
    a->tail = (full < st->G && chunk == chunks - 1) ? 1 : 0;
    return true;
}

bool sim_handle(const echo_state* st) { return st && st->rank < 0; }
bool rank_handle(const echo_state* st) { return st && st->rank >= 0; }

int set_device(const echo_state* st) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return ECHO_ECUDA;
    if (cur != st->device && cudaSetDevice(st->device) != cudaSuccess) return ECHO_ECUDA;
    return ECHO_OK;
}

}  // namespace

extern "C" {

size_t echo_state_bytes(int64_t n, int P, int group) {
    echo_layout L;
    return layout(n, P, group, 4, 4, &L) ? (size_t)L.state_bytes : 0;
}

size_t echo_workspace_bytes(int64_t n, int P, int group, int max_bits) {
    echo_layout L;
    return layout(n, P, group, max_bits, valid_bits(max_bits) ? max_bits : 0, &L) ? (size_t)L.workspace_bytes : 0;
}

int echo_query_layout(int64_t n, int P, int group, int max_bits, int bits, echo_layout* out) {
    if (!out) return ECHO_EINVAL;
    echo_layout L;
    if (!layout(n, P, group, max_bits, bits, &L)) return ECHO_EINVAL;
    *out = L;
    return ECHO_OK;
}

int echo_init_state(echo_state** out, int64_t n, int P, int group, int max_bits, void* state_dev,
                    void* workspace_dev, echo_stream_t stream) {
    echo_layout L;
    if (!out || !layout(n, P, group, max_bits, max_bits, &L)) return ECHO_EINVAL;
    if (!workspace_dev || !aligned(workspace_dev, kAlign)) return ECHO_EINVAL;
    if (state_dev && !aligned(state_dev, 16)) return ECHO_EINVAL;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ECHO_ECUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ECHO_ECUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (state_dev && cudaMemsetAsync(state_dev, 0, L.state_bytes, s) != cudaSuccess) return ECHO_ECUDA;
    if (cudaMemsetAsync(static_cast<uint8_t*>(workspace_dev) + L.flags_offset, 0, kAlign, s) != cudaSuccess)
        return ECHO_ECUDA;
    echo_state* st = new (std::nothrow) echo_state;
    if (!st) return ECHO_EINVAL;
    st->n = n;
    st->P = P;
    st->group = group;
    st->max_bits = max_bits;
    st->G = L.groups;
    st->S = L.state_stride;
    st->state = static_cast<float*>(state_dev);
    st->workspace = static_cast<uint8_t*>(workspace_dev);
    st->device = dev;
    st->sm_count = sms;
    st->quantizer = ECHO_QUANT_DIRECTED;
    st->have_events = false;
    st->rank = -1;
    st->wait_ns = kDefaultWaitNs;
    *out = st;
    return ECHO_OK;
}

int echo_set_wait_limit(echo_state* st, uint32_t limit_us) {
    if (!st || limit_us < kMinWaitUs || limit_us > kMaxWaitUs) return ECHO_EINVAL;
    st->wait_ns = 1000ull * limit_us;
    return ECHO_OK;
}

uint32_t echo_get_wait_limit(const echo_state* st) {
    return st ? (uint32_t)(st->wait_ns / 1000ull) : 0u;
}

int echo_set_quantizer(echo_state* st, int quantizer) {
    if (!st) return ECHO_EINVAL;
    if (quantizer != ECHO_QUANT_DIRECTED && quantizer != ECHO_QUANT_NEAREST && quantizer != ECHO_QUANT_INT_ZERO)
        return ECHO_EINVAL;
    st->quantizer = quantizer;
    return ECHO_OK;
}

int echo_phase_quantize(const void* const* inputs, echo_state* st, int bits, float eta, float alpha_long,
                        float alpha_short, float w, echo_stream_t stream) {
    if (!sim_handle(st) || !inputs || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_args(st, bits, inputs, nullptr, eta, alpha_long, alpha_short, w, &a)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    if (st->P < 2) return ECHO_OK;
    return launch(Stage::Quantize, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_phase_reduce(const void* const* inputs, void* const* outputs, echo_state* st, int bits, float eta,
                      float alpha_long, float alpha_short, float w, echo_stream_t stream) {
    if (!sim_handle(st) || !inputs || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    if (st->P == 1 && !outputs) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_args(st, bits, inputs, outputs, eta, alpha_long, alpha_short, w, &a)) return ECHO_EINVAL;
    a.write_outputs = outputs != nullptr;
    if (int rc = set_device(st)) return rc;
    return launch(Stage::Reduce, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_phase_gather(void* const* outputs, echo_state* st, int bits, echo_stream_t stream) {
    if (!sim_handle(st) || !outputs || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_args(st, bits, nullptr, outputs, 0.0f, 0.0f, 0.0f, 0.0f, &a)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    if (st->P < 2) return ECHO_OK;
    return launch(Stage::Gather, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_allreduce_sim(const void* const* inputs, void* const* outputs, echo_state* st, int64_t n, int P, int bits,
                       int group, float eta, float alpha_long, float alpha_short, float w, echo_stream_t stream) {
    if (!sim_handle(st) || !inputs || !outputs) return ECHO_EINVAL;
    if (n != st->n || P != st->P || group != st->group) return ECHO_EINVAL;
    if (!valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_args(st, bits, inputs, outputs, eta, alpha_long, alpha_short, w, &a)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    a.write_outputs = 1;   // the owner's pass decodes into every output (phase 4)
    if (P >= 2) {
        if (int rc = launch(Stage::Quantize, bits, a, st, s)) return rc;
    }
    return launch(Stage::Reduce, bits, a, st, s, P >= 2);
}

int echo_allreduce_sim_range(const void* const* inputs, void* const* outputs, echo_state* st, int64_t n, int P,
                             int bits, int group, float eta, float alpha_long, float alpha_short, float w,
                             int64_t group_begin, int64_t group_end, echo_stream_t stream) {
    if (!sim_handle(st) || !inputs || !outputs) return ECHO_EINVAL;
    if (n != st->n || P != st->P || group != st->group) return ECHO_EINVAL;
    if (!valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    if (group_begin < 0 || group_end < group_begin || group_end > st->G) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_args(st, bits, inputs, outputs, eta, alpha_long, alpha_short, w, &a)) return ECHO_EINVAL;
    if (group_begin == group_end) return ECHO_OK;
    if (int rc = set_device(st)) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    set_window(&a, st, group_begin, group_end);
    a.write_outputs = 1;
    if (P >= 2) {
        if (int rc = launch(Stage::Quantize, bits, a, st, s)) return rc;
    }
    return launch(Stage::Reduce, bits, a, st, s, P >= 2);
}

int echo_allreduce_sim_host(const void* const* host_inputs, void* host_output, void* const* inputs,
                            void* const* outputs, echo_state* st, int64_t n, int P, int bits, int group, float eta,
                            float alpha_long, float alpha_short, float w, int64_t chunk_groups,
                            echo_stream_t stream, echo_stream_t copy_in, echo_stream_t copy_out) {
    if (!sim_handle(st) || !host_inputs || !inputs || !outputs) return ECHO_EINVAL;
    if (n != st->n || P != st->P || group != st->group) return ECHO_EINVAL;
    if (!valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    if (chunk_groups < 0) return ECHO_EINVAL;
    for (int r = 0; r < P; ++r)
        if (!host_inputs[r]) return ECHO_EINVAL;
    echo_dev::Args probe;
    if (!make_args(st, bits, inputs, outputs, eta, alpha_long, alpha_short, w, &probe)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    if (!st->have_events) {
        for (int i = 0; i < 3; ++i) {
            if (cudaEventCreateWithFlags(&st->ev[i], cudaEventDisableTiming) != cudaSuccess) {
                for (int k = 0; k < i; ++k) cudaEventDestroy(st->ev[k]);
                return ECHO_ECUDA;
            }
        }
        st->have_events = true;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t cin = reinterpret_cast<cudaStream_t>(copy_in);
    cudaStream_t cout = reinterpret_cast<cudaStream_t>(copy_out);
    cudaEvent_t ev_start = st->ev[0], ev_in = st->ev[1], ev_done = st->ev[2];
    const int64_t G = st->G;
    const int64_t chunk = chunk_groups > 0 ? chunk_groups : (G + 15) / 16;
    // the copy streams start after everything already on `stream`
    if (cudaEventRecord(ev_start, s) != cudaSuccess) return ECHO_ECUDA;
    if (cudaStreamWaitEvent(cin, ev_start, 0) != cudaSuccess) return ECHO_ECUDA;
    if (host_output && cudaStreamWaitEvent(cout, ev_start, 0) != cudaSuccess) return ECHO_ECUDA;
    for (int64_t c0 = 0; c0 < G; c0 += chunk) {
        const int64_t c1 = c0 + chunk < G ? c0 + chunk : G;
        const int64_t e0 = c0 * group, e1 = c1 * group < n ? c1 * group : n;
        const size_t bytes = (size_t)(e1 - e0) * 2;
        for (int r = 0; r < P; ++r) {
            if (cudaMemcpyAsync(static_cast<uint16_t*>(inputs[r]) + e0,
                                static_cast<const uint16_t*>(host_inputs[r]) + e0, bytes, cudaMemcpyHostToDevice,
                                cin) != cudaSuccess)
                return ECHO_ECUDA;
        }
        // a wait binds to the event's latest record, so one event serves every chunk
        if (cudaEventRecord(ev_in, cin) != cudaSuccess) return ECHO_ECUDA;
        if (cudaStreamWaitEvent(s, ev_in, 0) != cudaSuccess) return ECHO_ECUDA;
        if (int rc = echo_allreduce_sim_range(inputs, outputs, st, n, P, bits, group, eta, alpha_long, alpha_short,
                                              w, c0, c1, stream))
            return rc;
        if (host_output) {
            if (cudaEventRecord(ev_done, s) != cudaSuccess) return ECHO_ECUDA;
            if (cudaStreamWaitEvent(cout, ev_done, 0) != cudaSuccess) return ECHO_ECUDA;
            if (cudaMemcpyAsync(static_cast<uint16_t*>(host_output) + e0, static_cast<const uint16_t*>(outputs[0]) + e0,
                                bytes, cudaMemcpyDeviceToHost, cout) != cudaSuccess)
                return ECHO_ECUDA;
        }
    }
    // `stream` continues once the last result has reached the host
    if (host_output) {
        if (cudaEventRecord(ev_done, cout) != cudaSuccess) return ECHO_ECUDA;
        if (cudaStreamWaitEvent(s, ev_done, 0) != cudaSuccess) return ECHO_ECUDA;
    }
    return ECHO_OK;
}

int echo_query_rank_layout(int64_t n, int P, int rank, int group, int max_bits, int bits, echo_rank_layout* out) {
    if (!out) return ECHO_EINVAL;
    echo_rank_layout L;
    if (!rank_layout(n, P, rank, group, max_bits, bits, &L)) return ECHO_EINVAL;
    *out = L;
    return ECHO_OK;
}

int echo_init_rank(echo_state** out, int64_t n, int P, int rank, int group, int max_bits, void* state_dev,
                   void* workspace_dev, echo_stream_t stream) {
    echo_rank_layout L;
    if (!out || !rank_layout(n, P, rank, group, max_bits, max_bits, &L)) return ECHO_EINVAL;
    if (!workspace_dev || !aligned(workspace_dev, kAlign)) return ECHO_EINVAL;
    if (state_dev && !aligned(state_dev, 16)) return ECHO_EINVAL;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ECHO_ECUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ECHO_ECUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (state_dev && cudaMemsetAsync(state_dev, 0, L.state_bytes, s) != cudaSuccess) return ECHO_ECUDA;
    // the flag word, and the payload buffers: padding the exchange never
    // writes is then defined
    if (cudaMemsetAsync(workspace_dev, 0, L.workspace_bytes, s) != cudaSuccess) return ECHO_ECUDA;
    echo_state* st = new (std::nothrow) echo_state;
    if (!st) return ECHO_EINVAL;
    st->n = n;
    st->P = P;
    st->group = group;
    st->max_bits = max_bits;
    st->G = L.groups;
    st->S = L.groups * group;
    st->state = static_cast<float*>(state_dev);
    st->workspace = static_cast<uint8_t*>(workspace_dev);
    st->device = dev;
    st->sm_count = sms;
    st->quantizer = ECHO_QUANT_DIRECTED;
    st->have_events = false;
    st->rank = rank;
    st->wait_ns = kDefaultWaitNs;
    *out = st;
    return ECHO_OK;
}

int echo_rank_quantize_chunk(const void* x, echo_state* st, int bits, float eta, float alpha_long,
                             float alpha_short, float w, int chunk, int chunks, echo_stream_t stream) {
    if (!rank_handle(st) || !x || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_rank_args(st, bits, RankPhase::Quantize, x, nullptr, eta, alpha_long, alpha_short, w, &a))
        return ECHO_EINVAL;
    if (!set_chunk(&a, st, chunk, chunks)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    if (st->P < 2) return ECHO_OK;
    return launch(Stage::Quantize, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_rank_reduce_chunk(const void* x, void* out, echo_state* st, int bits, float eta, float alpha_long,
                           float alpha_short, float w, int chunk, int chunks, echo_stream_t stream) {
    if (!rank_handle(st) || !x || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    if (st->P == 1 && !out) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_rank_args(st, bits, RankPhase::Reduce, x, st->P == 1 ? out : nullptr, eta, alpha_long, alpha_short,
                        w, &a))
        return ECHO_EINVAL;
    if (!set_chunk(&a, st, chunk, chunks)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    return launch(Stage::Reduce, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_rank_decode_chunk(void* out, echo_state* st, int bits, int chunk, int chunks, echo_stream_t stream) {
    if (!rank_handle(st) || !out || !valid_bits(bits) || bits > st->max_bits) return ECHO_EINVAL;
    echo_dev::Args a;
    if (!make_rank_args(st, bits, RankPhase::Decode, nullptr, out, 0.0f, 0.0f, 0.0f, 0.0f, &a)) return ECHO_EINVAL;
    if (!set_chunk(&a, st, chunk, chunks)) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    if (st->P < 2) return ECHO_OK;
    return launch(Stage::Gather, bits, a, st, reinterpret_cast<cudaStream_t>(stream));
}

int echo_rank_quantize(const void* x, echo_state* st, int bits, float eta, float alpha_long, float alpha_short,
                       float w, echo_stream_t stream) {
    return echo_rank_quantize_chunk(x, st, bits, eta, alpha_long, alpha_short, w, 0, 1, stream);
}

int echo_rank_reduce(const void* x, void* out, echo_state* st, int bits, float eta, float alpha_long,
                     float alpha_short, float w, echo_stream_t stream) {
    return echo_rank_reduce_chunk(x, out, st, bits, eta, alpha_long, alpha_short, w, 0, 1, stream);
}

int echo_rank_decode(void* out, echo_state* st, int bits, echo_stream_t stream) {
    return echo_rank_decode_chunk(out, st, bits, 0, 1, stream);
}

int echo_query_chunk(int64_t n, int P, int group, int owner, int chunk, int chunks, int64_t* first,
                     int64_t* count) {
    if (!first || !count || !valid_sizes(n, P, group) || owner < 0 || owner >= P) return ECHO_EINVAL;
    if (chunks < 1 || chunks > ECHO_MAX_CHUNKS || chunk < 0 || chunk >= chunks) return ECHO_EINVAL;
    const int64_t G = (n + group - 1) / group;
    const int64_t len = (int64_t)(owner + 1) * G / P - (int64_t)owner * G / P;
    const int64_t b = (int64_t)chunk * len / chunks, e = (int64_t)(chunk + 1) * len / chunks;
    *first = b;
    *count = e - b;
    return ECHO_OK;
}

namespace {

// SM count of the current device, looked up once per device.
int device_sms(int* dev_out) {
    static int sms[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (sms[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        sms[dev] = c;
    }
    *dev_out = dev;
    return sms[dev];
}

}  // namespace

int echo_bf16_allreduce_sim(const void* const* inputs, void* const* outputs, int64_t n, int P,
                            echo_stream_t stream) {
    if (!inputs || !outputs || n < 1 || n >= kMaxN || P < 1 || P > ECHO_MAX_RANKS) return ECHO_EINVAL;
    echo_dev::Args a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < P; ++r) {
        if (!inputs[r] || !outputs[r] || !aligned(inputs[r], 16) || !aligned(outputs[r], 16)) return ECHO_EINVAL;
        a.in[r] = static_cast<const uint16_t*>(inputs[r]);
        a.out[r] = static_cast<uint16_t*>(outputs[r]);
    }
    a.n = n;
    a.P = P;
    if (g_fail_launches.load(std::memory_order_relaxed)) return ECHO_ECUDA;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms == 0) return ECHO_ECUDA;
    static int per_sm[kMaxDevices];
    if (per_sm[dev] == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, echo_dev::k_bf16_allreduce_sim, echo_dev::kBf16Threads,
                                                          0) != cudaSuccess || b < 1)
            b = 1;
        per_sm[dev] = b;
    }
    const int64_t need = (n / 8 + echo_dev::kBf16Threads - 1) / echo_dev::kBf16Threads;
    const int grid = (int)(need < (int64_t)sms * per_sm[dev] ? (need > 0 ? need : 1) : (int64_t)sms * per_sm[dev]);
    echo_dev::k_bf16_allreduce_sim<<<grid, echo_dev::kBf16Threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
    return cuda_status(cudaGetLastError());
}

int echo_background_traffic(const void* src, void* dst, size_t bytes, uint32_t duty_permille, uint32_t period_us,
                            uint32_t duration_us, unsigned long long* moved_dev, echo_stream_t stream) {
    if (!src || !dst || !aligned(src, 16) || !aligned(dst, 16) || bytes < (size_t)echo_dev::kBgChunk ||
        bytes % echo_dev::kBgChunk != 0)
        return ECHO_EINVAL;
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
    if (s0 < d0 + bytes && d0 < s0 + bytes) return ECHO_EINVAL;   // overlapping buffers
    if (duty_permille > 1000 || period_us < 10 || period_us > 1000000 || duration_us < 1 ||
        duration_us > 60000000u)
        return ECHO_EINVAL;
    if (moved_dev && !aligned(moved_dev, 8)) return ECHO_EINVAL;
    if (duty_permille == 0) return ECHO_OK;   // no traffic: nothing to launch
    if (g_fail_launches.load(std::memory_order_relaxed)) return ECHO_ECUDA;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms == 0) return ECHO_ECUDA;
    const unsigned long long period_ns = 1000ull * period_us;
    const unsigned long long on_ns = period_ns * duty_permille / 1000ull;
    static int smem_set[kMaxDevices];
    if (!smem_set[dev]) {
        if (cudaFuncSetAttribute(echo_dev::k_background_traffic, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 echo_dev::kBgSmem) != cudaSuccess)
            return ECHO_ECUDA;
        smem_set[dev] = 1;
    }
    echo_dev::k_background_traffic<<<sms, 32, echo_dev::kBgSmem, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), (long long)(bytes / echo_dev::kBgChunk), on_ns,
        period_ns, 1000ull * duration_us, moved_dev);
    return cuda_status(cudaGetLastError());
}

int echo_inject_launch_failure(int enable) {
    return g_fail_launches.exchange(enable ? 1 : 0);
}

int echo_check_watchdog(echo_state* st, uint32_t limit_us, echo_stream_t stream) {
    if (!st || limit_us > 10000000u) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    const unsigned long long limit_ns = limit_us == 0 ? st->wait_ns : 1000ull * limit_us;
    echo_dev::k_watchdog_check<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<uint32_t*>(st->workspace), limit_ns);
    return cuda_status(cudaGetLastError());
}

int echo_get_status(echo_state* st, echo_stream_t stream, uint32_t* device_flags) {
    if (!st) return ECHO_EINVAL;
    if (int rc = set_device(st)) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t flags = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ECHO_ECUDA;
    if (cudaMemcpy(&flags, st->workspace, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess) return ECHO_ECUDA;
    if (cudaMemset(st->workspace, 0, sizeof(flags)) != cudaSuccess) return ECHO_ECUDA;
    if (device_flags) *device_flags = flags;
    if (flags & ECHO_FLAG_TIMEOUT) return ECHO_ETIMEOUT;
    return (flags & ECHO_FLAG_RANGE) ? ECHO_ERANGE : ECHO_OK;
}

int echo_free(echo_state* st) {
    if (st && st->have_events) {
        int cur = -1;
        const bool switched = cudaGetDevice(&cur) == cudaSuccess && cur != st->device &&
                              cudaSetDevice(st->device) == cudaSuccess;
        for (cudaEvent_t e : st->ev) cudaEventDestroy(e);
        if (switched) cudaSetDevice(cur);
    }
    delete st;
    return ECHO_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation entry point: payloads and flag word in a fixed scratch array.

// Scratch of echo_allreduce_sim_noalloc. In host code this name is only a
// stand-in for the symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ECHO_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
uint8_t* g_noalloc_ptr[kNoallocMaxDevices];   // device address of the scratch, per device
int g_noalloc_sms[kNoallocMaxDevices];

// Once per device, with that device current: the scratch's device address and
// the SM count.
int noalloc_setup(int dev, uint8_t** ptr, int* sms) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return ECHO_ECUDA;
        int count = 0;
        if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ECHO_ECUDA;
        g_noalloc_sms[dev] = count;
        g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *ptr = g_noalloc_ptr[dev];
    *sms = g_noalloc_sms[dev];
    return ECHO_OK;
}

}  // namespace

extern "C" {

int echo_allreduce_sim_noalloc(const void* const* inputs, void* const* outputs, void* state_dev, int64_t n, int P,
                               int bits, int group, float eta, float alpha_long, float alpha_short, float w,
                               uint32_t* flags_out, echo_stream_t stream) {
    if (!inputs || !outputs) return ECHO_EINVAL;
    echo_layout L;
    if (!layout(n, P, group, bits, bits, &L)) return ECHO_EINVAL;
    if (!valid_feedback(eta, alpha_long, alpha_short, w)) return ECHO_EINVAL;
    if (state_dev && !aligned(state_dev, 16)) return ECHO_EINVAL;
    if (L.workspace_bytes > (uint64_t)ECHO_NOALLOC_SCRATCH_BYTES) return ECHO_ENOSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return ECHO_ECUDA;
    uint8_t* scratch = nullptr;
    int sms = 0;
    if (int rc = noalloc_setup(dev, &scratch, &sms)) return rc;
    echo_state st;   // on the stack: describes the call, owns nothing
    st.n = n;
    st.P = P;
    st.group = group;
    st.max_bits = bits;
    st.G = L.groups;
    st.S = L.state_stride;
    st.state = static_cast<float*>(state_dev);
    st.workspace = scratch;
    st.device = dev;
    st.sm_count = sms;
    st.quantizer = ECHO_QUANT_DIRECTED;
    st.have_events = false;
    st.rank = -1;
    st.wait_ns = kDefaultWaitNs;
    echo_dev::Args a;
    if (!make_args(&st, bits, inputs, outputs, eta, alpha_long, alpha_short, w, &a)) return ECHO_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch + L.flags_offset, 0, sizeof(uint32_t), s) != cudaSuccess) return ECHO_ECUDA;
    a.write_outputs = 1;
    if (P >= 2) {
        if (int rc = launch(Stage::Quantize, bits, a, &st, s)) return rc;
    }
    if (int rc = launch(Stage::Reduce, bits, a, &st, s)) return rc;
    if (flags_out) {
        uint32_t f = 0;
        if (cudaStreamSynchronize(s) != cudaSuccess) return ECHO_ECUDA;
        if (cudaMemcpy(&f, scratch + L.flags_offset, sizeof(f), cudaMemcpyDeviceToHost) != cudaSuccess)
            return ECHO_ECUDA;
        *flags_out = f;
        if (f & ECHO_FLAG_TIMEOUT) return ECHO_ETIMEOUT;
        if (f & ECHO_FLAG_RANGE) return ECHO_ERANGE;
    }
    return ECHO_OK;
}

const char* echo_status_string(int status) {
    switch (status) {
        case ECHO_OK: return "ok";
        case ECHO_EINVAL: return "invalid argument";
        case ECHO_ECUDA: return "CUDA error";
        case ECHO_ERANGE: return "value outside the fp16 parameter range";
        case ECHO_ETIMEOUT: return "device wait timed out";
        case ECHO_ENOSPACE: return "message too large for the no-allocation scratch (ECHO_NOALLOC_SCRATCH_BYTES)";
    }
    return "unknown status";
}

}  // extern "C"
