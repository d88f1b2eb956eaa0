/*
 * echo.h -- C ABI of the single-GPU simulation of Echo's 4-bit
 * error-compensated all-reduce.
 *
 * The method (sources, in prose only -- the pages print no code):
 *   [ABS] "Echo: Error-Compensated 4-Bit Tensor-Parallel Communication for
 *         LLM Training and Inference" (arXiv 2610.14277), abstract;
 *   [EXP] the explainer "テンソル並列の通信を4bitに圧縮する「Echo」",
 *         sections "Echoの仕組み①" (mechanism 1: the all-reduce becomes an
 *         all-to-all of 4-bit non-owned segments, a high-precision sum at each
 *         segment's owner and a 4-bit all-gather of the requantized sum),
 *         "Echoの仕組み②" (mechanism 2: the residuals the ranks keep sum to
 *         minus the injected error; a long and a short moving average of them
 *         are added back into the next call's input, fused into the entry
 *         pass), "実測性能と精度" (an 8-bit mode for early layers) and
 *         "よくある質問" (FAQ: the payload is 4-bit integers plus
 *         half-precision parameters).
 *
 * One call of echo_allreduce_sim computes, for P virtual ranks whose bf16
 * partial sums all sit in the memory of ONE GPU, the five phases:
 *   1. feedback injection  x' = x + eta * (w * e_short + (1 - w) * e_long)
 *   2. per-group asymmetric quantization of every rank's NON-owned groups
 *      (fp16 scale s and zero z, codes packed two per byte): the all-to-all
 *      payload, written to device memory;
 *   3. at each group's owner: binary32 sum, in rank order 0..P-1, of its own
 *      unquantized x' and the P-1 dequantized payloads, requantized into the
 *      all-gather payload;
 *   4. every rank dequantizes the gathered payload into its bf16 output;
 *   5. the residuals (non-owner: x' - x_hat; owner: sum - y) update both
 *      EMAs:  e <- (1 - alpha) * e + alpha * rho.
 * The "transport" is the payload buffers in device memory; nothing crosses
 * GPUs. The exact arithmetic (directed fp16 rounding of z and s, half-to-even
 * codes, no fused multiply-add) is stated at echo_allreduce_sim below.
 *
 * Memory: the library never allocates device memory. The caller owns the P
 * input and output buffers, the EMA state and a workspace; their sizes come
 * from echo_state_bytes / echo_workspace_bytes. All work is enqueued on the
 * caller's stream. Every function is host-callable, returns an echo_status
 * and does not block unless stated.
 */
#ifndef ECHO_H
#define ECHO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility when the library is built with
 * hidden visibility. */
#if defined(__GNUC__)
#define ECHO_API __attribute__((visibility("default")))
#else
#define ECHO_API
#endif

/* Largest number of virtual ranks a call accepts. */
#define ECHO_MAX_RANKS 64

/* Sticky device flags read by echo_get_status. */
#define ECHO_FLAG_RANGE 1u   /* a quantized group (or a P == 1 output) held a
                                value outside [-65504, 65504] or a NaN: the
                                fp16 parameters cannot describe it; outputs
                                and state of that group are unspecified */
#define ECHO_FLAG_TIMEOUT 2u /* a bounded device-side wait (between the
                                bulk-copy producer and the compute warps of
                                a kernel) expired; that call's results are
                                unspecified */

typedef enum echo_status {
    ECHO_OK = 0,
    ECHO_EINVAL = 1,     /* bad argument; nothing was enqueued */
    ECHO_ECUDA = 2,      /* a CUDA runtime call or kernel launch failed */
    ECHO_ERANGE = 3,     /* returned by echo_get_status when ECHO_FLAG_RANGE is set */
    ECHO_ETIMEOUT = 4,   /* returned by echo_get_status when ECHO_FLAG_TIMEOUT is set */
    ECHO_ENOSPACE = 5    /* echo_allreduce_sim_noalloc: the message needs more
                            scratch than ECHO_NOALLOC_SCRATCH_BYTES */
} echo_status;

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* echo_stream_t;

/* Opaque host-side handle: sizes, the caller's state/workspace pointers and
 * the launch configuration. It owns no device memory. */
typedef struct echo_state echo_state;

/* Byte offsets inside the workspace for a call with `bits`, and sizes.
 *   flags          uint32 sticky flag word (ECHO_FLAG_*)
 *   a2a codes      [P][G][code_bytes]  slot [r][j]: rank r's packed codes of
 *                  group j, sent to owner(j); the owner's own slot is unused
 *   a2a params     [P][G] uint32: fp16 bits of s in the low half, of z in the
 *                  high half (little-endian: {s, z} as two uint16)
 *   gather codes   [G][code_bytes]   the owner's requantized sum of group j
 *   gather params  [G] uint32        as above
 * Codes of a 4-bit group: element 2i in the low nibble, 2i+1 in the high
 * nibble of byte i; 8-bit: one byte per element; a partial last group is
 * padded with code 0. Group j covers elements [j*group, min(n, (j+1)*group))
 * of the flattened message; owner(j) = the s with
 * floor(s*G/P) <= j < floor((s+1)*G/P). */
typedef struct echo_layout {
    int64_t groups;              /* G = ceil(n / group) */
    int64_t state_stride;        /* S = G * group floats per EMA per rank */
    uint64_t code_bytes;         /* group * bits / 8 */
    uint64_t flags_offset;
    uint64_t a2a_codes_offset;
    uint64_t a2a_params_offset;
    uint64_t gather_codes_offset;
    uint64_t gather_params_offset;
    uint64_t workspace_bytes;    /* for max_bits */
    uint64_t state_bytes;
} echo_layout;

/* Bytes of EMA state: float32 [P][2][S], S = ceil(n/group)*group; [r][0] is
 * rank r's long EMA, [r][1] its short EMA; element k of the message at
 * offset k (the padding past n is never read or written). 0 on bad sizes. */
ECHO_API size_t echo_state_bytes(int64_t n, int P, int group);

/* Bytes of workspace for calls with bits <= max_bits. 0 on bad sizes. */
ECHO_API size_t echo_workspace_bytes(int64_t n, int P, int group, int max_bits);

/* Fill *out for a call with `bits` (<= max_bits). ECHO_EINVAL on bad sizes. */
ECHO_API int echo_query_layout(int64_t n, int P, int group, int max_bits, int bits, echo_layout* out);

/*
 * Create a handle for messages of n elements per rank over P ranks.
 *   n          1 <= n < 2^40
 *   P          1..ECHO_MAX_RANKS
 *   group      32, 64, 128 or 256 elements per quantization group
 *   max_bits   4 or 8: the largest `bits` later calls will use
 *   state_dev  device pointer to echo_state_bytes(n, P, group) bytes, 16-byte
 *              aligned, or NULL for "no feedback" (x' = x, no state traffic)
 *   workspace_dev  device pointer to echo_workspace_bytes(...) bytes,
 *              256-byte aligned
 *   stream     the EMAs (if any) and the flag word are zeroed on it
 * The caller keeps ownership of both buffers and must keep them alive until
 * echo_free. Returns ECHO_EINVAL (nothing enqueued, *out untouched) or
 * ECHO_ECUDA.
 */
ECHO_API int echo_init_state(echo_state** out, int64_t n, int P, int group, int max_bits,
                    void* state_dev, void* workspace_dev, echo_stream_t stream);

/*
 * Quantizer forms. The Echo explainer (section "Echoの仕組み①", mechanism 1)
 * names an asymmetric, zero-point-aware group quantizer with half-precision
 * parameters (section "よくある質問", FAQ) and fixes neither how those
 * parameters round nor whether the zero is a float or an integer; the
 * ablations compare three readings. Every form ships `bits`-bit codes plus
 * one 32-bit parameter word per group (low half: fp16 step s).
 *   ECHO_QUANT_DIRECTED  (default) z = fp16 rounded toward -inf from the
 *        group minimum, s = fp16 rounded toward +inf from (max - z) / Q;
 *        code = rint((v - z) / s); value = code * s + z. High half: fp16 z.
 *   ECHO_QUANT_NEAREST   z and s = (max - min) / Q both rounded to nearest;
 *        codes clamped to [0, Q]; value = code * s + z. High half: fp16 z.
 *   ECHO_QUANT_INT_ZERO  integer zero point: the range is widened to include
 *        0 (lo = min(min, 0), hi = max(max, 0)); s = fp16 rounded up from
 *        (hi - lo) / Q; zp = clamp(rint(-lo / s), 0, Q);
 *        code = clamp(rint(v / s) + zp, 0, Q); value = (code - zp) * s, so 0
 *        is always exactly representable. High half: zp as an integer.
 * (Divisions are binary32 multiplications by 1/s rounded to nearest; rint
 * rounds half to even.)
 */
#define ECHO_QUANT_DIRECTED 0
#define ECHO_QUANT_NEAREST 1
#define ECHO_QUANT_INT_ZERO 2

/*
 * Select the quantizer form for the calls that use `st` from now on (the
 * handle starts with ECHO_QUANT_DIRECTED; echo_allreduce_sim_noalloc always
 * uses it). Both stages of a call use the same form. Host-only: enqueues
 * nothing. ECHO_EINVAL for a NULL handle or an unknown form.
 */
ECHO_API int echo_set_quantizer(echo_state* st, int quantizer);

/*
 * One all-reduce call over the P virtual ranks (phases 1-5 above).
 *   inputs     host array of P device pointers, each to n bf16 values
 *              (16-byte aligned): rank r's partial sum
 *   outputs    host array of P device pointers, each to n bf16 values
 *              (16-byte aligned): rank r's copy of the reduced result. An
 *              output may be the same buffer as an input; other overlaps are
 *              undefined.
 *   st         handle from echo_init_state; n, P and group must match it
 *   bits       4 (INT4) or 8 (the early-site 8-bit mode), <= the handle's
 *              max_bits
 *   eta        feedback gain, finite
 *   alpha_long, alpha_short   EMA rates in [0, 1]
 *   w          weight of the short EMA in the compensation, in [0, 1]
 *   stream     CUDA stream; the call is asynchronous on it. For P >= 2 it is two
 *              kernels (the non-owners' quantize pass, then the owners'
 *              pass); the second is a programmatic dependent launch of the
 *              first, so it may start while the first drains, but it reads
 *              nothing the first writes before that kernel has completed.
 *              Towards other work on the stream the call is ordered as usual.
 * Arithmetic (binary32, round-to-nearest, no contraction into fused
 * multiply-add): c = eta*(w*e_short + (1-w)*e_long), x' = float(x) + c
 * (x' = float(x) without state); per group mn = min + 0, mx = max + 0,
 * z = fp16 rounded toward -inf of mn, s = fp16 rounded toward +inf of
 * (mx - z)/Q with Q = 2^bits - 1, code = clamp(rint_even((v - z) * (1/s)),
 * 0, Q) (all 0 when s == 0), x_hat = code*s + z; the owner sums in rank
 * order; y = bf16 round-to-nearest-even of the requantized sum (of x' when
 * P == 1); each EMA e <- (1-alpha)*e + alpha*rho.
 * Errors: ECHO_EINVAL when an argument is out of range, a pointer is NULL
 * or misaligned, or n/P/group differ from the handle (nothing is enqueued);
 * ECHO_ECUDA when a launch fails. Data-dependent range violations do not
 * stop the call: they set ECHO_FLAG_RANGE (see echo_get_status).
 */
ECHO_API int echo_allreduce_sim(const void* const* inputs, void* const* outputs, echo_state* st,
                       int64_t n, int P, int bits, int group,
                       float eta, float alpha_long, float alpha_short, float w,
                       echo_stream_t stream);

/*
 * The phases one by one (same arguments and errors as echo_allreduce_sim):
 *   echo_phase_quantize  phases 1, 2 and 5 for every rank's non-owned groups:
 *                        writes the all-to-all payload and those EMAs
 *                        (does nothing when P == 1)
 *   echo_phase_reduce    phases 1, 3 and 5 for every group's owner: reads the
 *                        all-to-all payload, writes the all-gather payload
 *                        and the owners' EMAs. When `outputs` is given (it is
 *                        required when P == 1) the same pass also performs
 *                        phase 4: the owner decodes its requantized sum --
 *                        the very bits of the all-gather payload -- into all
 *                        P outputs. echo_allreduce_sim is echo_phase_quantize
 *                        followed by echo_phase_reduce with outputs.
 *   echo_phase_gather    phase 4 on its own: decodes the all-gather payload
 *                        into all P outputs (the same result; for callers
 *                        that ran echo_phase_reduce without outputs; does
 *                        nothing when P == 1)
 */
ECHO_API int echo_phase_quantize(const void* const* inputs, echo_state* st, int bits,
                        float eta, float alpha_long, float alpha_short, float w,
                        echo_stream_t stream);
ECHO_API int echo_phase_reduce(const void* const* inputs, void* const* outputs, echo_state* st, int bits,
                      float eta, float alpha_long, float alpha_short, float w,
                      echo_stream_t stream);
ECHO_API int echo_phase_gather(void* const* outputs, echo_state* st, int bits, echo_stream_t stream);

/*
 * echo_allreduce_sim restricted to the group columns [group_begin, group_end)
 * of the message: for every rank, groups j with group_begin <= j < group_end
 * (elements [j*group, min(n, (j+1)*group))), with the ownership of the WHOLE
 * message (owner(j) as documented at echo_layout). A group column -- group j
 * of every rank, its payload slots and its EMA entries -- is computed
 * independently of every other column in all five phases (the explainer's
 * mechanism 1 reduces each segment at its owner, group by group), so calls on
 * disjoint windows that together cover [0, G) give, bit for bit, the
 * outputs, payloads, EMAs and flags of one echo_allreduce_sim call, in any
 * order. Elements outside the window are neither read nor written. This lets
 * a caller run the all-reduce chunk by chunk while other chunks are still
 * being produced or copied (see echo_allreduce_sim_host).
 *   group_begin, group_end  0 <= group_begin <= group_end <= G
 *                           (G = ceil(n/group)); an empty window enqueues
 *                           nothing
 *   all other arguments     as for echo_allreduce_sim
 * Errors: those of echo_allreduce_sim; ECHO_EINVAL for a window out of range.
 */
ECHO_API int echo_allreduce_sim_range(const void* const* inputs, void* const* outputs, echo_state* st,
                             int64_t n, int P, int bits, int group,
                             float eta, float alpha_long, float alpha_short, float w,
                             int64_t group_begin, int64_t group_end, echo_stream_t stream);

/*
 * One all-reduce call whose P inputs start, and whose result ends, in host
 * memory: the library copies the inputs in, runs echo_allreduce_sim_range
 * chunk by chunk and copies the result out, overlapping the host-to-device
 * copies of later chunks, the kernels of the current chunk and the
 * device-to-host copy of earlier chunks on three streams. (The pages' own
 * kernel pipelines quantization with NVLink transfers; on one GPU the
 * transfers that remain are the host link's.) Results are bit-identical to
 * copying everything in, one echo_allreduce_sim call, and copying out.
 *   host_inputs  host array of P host pointers, each to n bf16 values
 *                (rank r's partial sum). Page-locked (pinned) memory is
 *                needed for the copies to overlap; pageable memory works but
 *                serializes them.
 *   host_output  host pointer to n bf16 values that receives the reduced
 *                result (identical on every rank; copied from outputs[0]),
 *                or NULL to leave the result on the device only
 *   inputs, outputs  the device buffers of echo_allreduce_sim; the inputs
 *                are overwritten with host_inputs, every output receives the
 *                result
 *   chunk_groups group columns per chunk, >= 1; 0 picks ceil(G / 16)
 *   stream       the kernels run on it; the call is ordered after earlier
 *                work on `stream`, and later work on `stream` waits until
 *                the result has reached host_output
 *   copy_in, copy_out  streams for the host-to-device and device-to-host
 *                copies (may equal `stream`, which gives up the overlap)
 *   all other arguments  as for echo_allreduce_sim
 * Asynchronous: the host buffers must stay valid, and host_output must not
 * be read, until `stream` has reached this point (synchronize it, or an
 * event recorded on it after the call). The first call on a handle creates
 * three CUDA events (no device memory), released by echo_free.
 * Errors: those of echo_allreduce_sim (nothing enqueued on ECHO_EINVAL);
 * ECHO_ECUDA when a copy, event or launch fails, in which case part of the
 * work may already be enqueued.
 */
ECHO_API int echo_allreduce_sim_host(const void* const* host_inputs, void* host_output, void* const* inputs,
                            void* const* outputs, echo_state* st, int64_t n, int P, int bits, int group,
                            float eta, float alpha_long, float alpha_short, float w, int64_t chunk_groups,
                            echo_stream_t stream, echo_stream_t copy_in, echo_stream_t copy_out);

/*
 * Synchronize `stream`, read the sticky flag word into *device_flags (may be
 * NULL) and clear it. Returns ECHO_ETIMEOUT when ECHO_FLAG_TIMEOUT was set,
 * else ECHO_ERANGE when ECHO_FLAG_RANGE was set, else ECHO_OK;
 * ECHO_ECUDA if the synchronization or copy fails.
 * Blocks the host.
 */
ECHO_API int echo_get_status(echo_state* st, echo_stream_t stream, uint32_t* device_flags);

/*
 * Limit of the kernels' bounded device-side waits for the later calls of a
 * handle (no counterpart on the pages; part of this library's failure
 * detection). Every wait of the bulk-copy pipelines (a consumer waiting for a
 * staged tile, the producer waiting for a free slot or for its own copies to
 * land) gives up after this long, sets ECHO_FLAG_TIMEOUT and ends the kernel
 * early; that call's results are then undefined. The default, 1 s, is far
 * above any wait of a healthy call; a caller that shares the GPU with other
 * contexts time-sliced for long periods may raise it.
 *   limit_us   1000 .. 60 000 000 (1 ms .. 60 s)
 * Host-only, takes effect at the handle's next launch. ECHO_EINVAL on a NULL
 * handle or a limit out of range (the setting is then unchanged).
 * echo_allreduce_sim_noalloc, which has no handle, always uses the default.
 */
ECHO_API int echo_set_wait_limit(echo_state* st, uint32_t limit_us);

/* The handle's wait limit in microseconds (0 for a NULL handle). */
ECHO_API uint32_t echo_get_wait_limit(const echo_state* st);

/*
 * Failure-detection self-check (no counterpart on the pages; part of this
 * library's error reporting). Launches one thread that waits, with the same
 * bounded wait the bulk-copy pipelines use, on a barrier that nothing ever
 * completes. After limit_us microseconds (1 .. 10^7; 0: the handle's wait
 * limit, see echo_set_wait_limit) the wait gives up, the kernel sets
 * ECHO_FLAG_TIMEOUT in st's flag word and returns; the next echo_get_status
 * returns ECHO_ETIMEOUT and the context stays usable.
 * Asynchronous on `stream`. ECHO_EINVAL on a NULL handle or a limit out of
 * range, ECHO_ECUDA when the launch fails.
 */
ECHO_API int echo_check_watchdog(echo_state* st, uint32_t limit_us, echo_stream_t stream);

/*
 * Fault-injection hook for tests of callers' error paths (no counterpart on
 * the pages; part of this library's failure detection). While enabled
 * (enable != 0), every call that would launch one of the all-reduce kernels
 * returns ECHO_ECUDA at that launch instead: the kernel is not launched;
 * work a call enqueues before its first launch (the host-buffer call's first
 * copies, the no-allocation call's flag clear) stays enqueued. Process-wide,
 * host-only; nothing on the GPU fails. Returns the previous setting (0 or 1).
 */
ECHO_API int echo_inject_launch_failure(int enable);

/* Size of the fixed scratch array used by echo_allreduce_sim_noalloc. It is
 * device memory that every GPU which loads this library holds until the
 * process exits. */
#define ECHO_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * echo_allreduce_sim for callers that cannot allocate device memory. The
 * pages describe no such variant; this entry point has no counterpart in the
 * paper.
 *
 * Who needs it: code that may not allocate device memory at the point where
 * it runs the all-reduce -- a process whose framework reserved the device
 * memory for its own pools at start-up (a serving engine that pre-allocates
 * its KV cache, say), or a latency-critical path that cannot afford the
 * implicit device-wide synchronization of cudaMalloc/cudaFree. Such callers
 * cannot provide the workspace echo_init_state needs. Here the all-to-all and
 * all-gather payloads and the flag word live in a fixed scratch array inside
 * this library (ECHO_NOALLOC_SCRATCH_BYTES, 16 MiB), there is no handle, and
 * nothing is allocated -- not by this call, not by the caller. The kernels and
 * the arithmetic are those of echo_allreduce_sim, so the results are
 * identical.
 *
 *   inputs, outputs, n, P, bits, group, eta, alpha_long, alpha_short, w,
 *   stream     as for echo_allreduce_sim
 *   state_dev  NULL (no feedback), or the caller's EMA state: device memory of
 *              echo_state_bytes(n, P, group) bytes, 16-byte aligned, in the
 *              layout documented at echo_state_bytes. The caller zeroes it
 *              before the first call and keeps it between calls.
 *   flags_out  NULL, or a host word that receives this call's ECHO_FLAG_*
 *              bits; when given, the call synchronizes `stream` before
 *              returning and maps the bits to its return code as
 *              echo_get_status does: ECHO_ETIMEOUT when ECHO_FLAG_TIMEOUT is
 *              set, else ECHO_ERANGE when ECHO_FLAG_RANGE is set. Without
 *              flags_out nothing reports a range or timeout failure of the
 *              call: there is no handle to query, and the next call clears
 *              the flag word.
 * Limit: the payloads of the message must fit the scratch:
 *   echo_query_layout(n, P, group, bits, bits).workspace_bytes, about
 *   (P + 1) * ceil(n / group) * (group * bits / 8 + 4) bytes, must not exceed
 *   ECHO_NOALLOC_SCRATCH_BYTES (for P = 8, 4 bits, groups of 128: up to about
 *   3.4 M elements per rank). A larger message returns ECHO_ENOSPACE before
 *   anything is enqueued.
 * Set-up: the first call on a device looks up, with that device current, the
 *   device address of the scratch array and the device's SM count, and keeps
 *   them for later calls. Make that first call on each device before any
 *   stream capture on it.
 * Sharing: all calls on a device use the same scratch, which keeps the last
 *   call's payloads; each call clears the flag word before its kernels run.
 *   Calls that overlap on the GPU (on streams with no ordering between them)
 *   race on the scratch and give undefined results: order them.
 * Errors: those of echo_allreduce_sim, plus ECHO_ENOSPACE; with flags_out,
 *   also ECHO_ERANGE and ECHO_ETIMEOUT (data-dependent, after the call ran).
 * Waits: the kernels' bounded waits use the default limit (1 s).
 */
ECHO_API int echo_allreduce_sim_noalloc(const void* const* inputs, void* const* outputs, void* state_dev,
                                        int64_t n, int P, int bits, int group, float eta, float alpha_long,
                                        float alpha_short, float w, uint32_t* flags_out, echo_stream_t stream);

/*
 * ------------------------------------------------------------------------
 * One rank of a multi-GPU call: one process (or one handle) per GPU, P ranks.
 *
 * The same restructured all-reduce ([EXP] mechanism 1) with the transport
 * between the phases done by the caller's collectives (NCCL through
 * torch.distributed, say) instead of shared device memory:
 *   1. echo_rank_quantize   phases 1, 2, 5 for this rank's non-owned groups:
 *                           fills its all-to-all send row
 *   2. all-to-all           (caller) send row -> every owner's receive rows
 *   3. echo_rank_reduce     phases 1, 3, 5 for this rank's own segment: sums
 *                           its x' and the P-1 received payloads in rank order,
 *                           requantizes into its all-gather send buffer
 *   4. all-gather           (caller) every rank's send buffer -> receive rows
 *   5. echo_rank_decode     phase 4: decodes every gathered segment into this
 *                           rank's output
 * The arithmetic is that of echo_allreduce_sim: P ranks running this
 * sequence produce, bit for bit, the simulation's outputs, payloads and EMA
 * state (rank r holding rows r of the simulation's [P][2][S] state).
 *
 * Workspace of one rank (byte offsets; code regions sized for max_bits, laid
 * out with code_bytes = group * bits / 8 of the call):
 *   send codes   [G][code_bytes], send params [G] (uint32 {s, z} words):
 *                this rank's payload for group j at j; the part for owner s
 *                is groups [seg_begin(s), seg_begin(s) + seg_groups(s)),
 *                i.e. seg_groups(s) * code_bytes bytes at
 *                seg_begin(s) * code_bytes (params: seg_groups(s) words at
 *                seg_begin(s)). The part for this rank itself is written and
 *                never read.
 *   recv codes   [P][seg_groups][code_bytes], recv params [P][seg_groups]:
 *                what rank r sent to this owner, at r * seg_groups groups.
 *                An all-to-all with these splits (send counts seg_groups(s),
 *                receive counts seg_groups of this rank from every rank) fills
 *                it; torch.distributed.all_to_all_single does.
 *   gsend codes  [seg_max][code_bytes], gsend params [seg_max]: this owner's
 *                requantized segment (the first seg_groups entries).
 *   grecv codes  [P][seg_max][code_bytes], grecv params [P][seg_max]: every
 *                owner's gsend, in rank order: an all-gather of gsend.
 * segment s = groups [floor(s G / P), floor((s + 1) G / P)); seg_max = the
 * largest segment.
 */
typedef struct echo_rank_layout {
    int64_t groups;               /* G = ceil(n / group) */
    int64_t seg_begin;            /* first group this rank owns */
    int64_t seg_groups;           /* groups this rank owns (may be 0 when G < P) */
    int64_t seg_max;              /* largest segment of any rank */
    uint64_t code_bytes;          /* group * bits / 8 */
    uint64_t flags_offset;
    uint64_t send_codes_offset;
    uint64_t send_params_offset;
    uint64_t recv_codes_offset;
    uint64_t recv_params_offset;
    uint64_t gsend_codes_offset;
    uint64_t gsend_params_offset;
    uint64_t grecv_codes_offset;
    uint64_t grecv_params_offset;
    uint64_t workspace_bytes;     /* for max_bits */
    uint64_t state_bytes;         /* this rank's two EMAs: float32 [2][S] */
} echo_rank_layout;

/* Fill *out for rank `rank` (0 <= rank < P) and a call with `bits`.
 * Host-only. ECHO_EINVAL on bad sizes. */
ECHO_API int echo_query_rank_layout(int64_t n, int P, int rank, int group, int max_bits, int bits,
                                    echo_rank_layout* out);

/*
 * Handle of one rank. Arguments as for echo_init_state, with
 *   rank       this rank, 0 <= rank < P
 *   state_dev  NULL (no feedback) or device memory of
 *              echo_query_rank_layout(...).state_bytes, 16-byte aligned:
 *              this rank's long EMA then short EMA (S floats each)
 *   workspace_dev  device memory of workspace_bytes, 256-byte aligned
 * The state and the whole workspace are zeroed on `stream`. The handle
 * serves only the echo_rank_* calls (and echo_set_quantizer,
 * echo_get_status, echo_check_watchdog, echo_free); the simulation's calls
 * return ECHO_EINVAL for it.
 */
ECHO_API int echo_init_rank(echo_state** out, int64_t n, int P, int rank, int group, int max_bits,
                            void* state_dev, void* workspace_dev, echo_stream_t stream);

/* Step 1 on this rank: x = its n bf16 inputs (device, 16-byte aligned).
 * Nothing to do when P == 1. Errors as for echo_allreduce_sim. */
ECHO_API int echo_rank_quantize(const void* x, echo_state* st, int bits, float eta, float alpha_long,
                                float alpha_short, float w, echo_stream_t stream);

/* Step 3 on this rank, after the all-to-all has filled its receive rows: x =
 * the same inputs as step 1. When P == 1 it also writes the result into
 * `out` (n bf16, required then); otherwise `out` is ignored (may be NULL). */
ECHO_API int echo_rank_reduce(const void* x, void* out, echo_state* st, int bits, float eta, float alpha_long,
                              float alpha_short, float w, echo_stream_t stream);

/* Step 5 on this rank, after the all-gather has filled its gathered rows:
 * writes the reduced result (n bf16) into `out`. Nothing to do when P == 1. */
ECHO_API int echo_rank_decode(void* out, echo_state* st, int bits, echo_stream_t stream);

/*
 * Chunked calls of one rank: the explainer ("Echoの仕組み①") hides
 * quantization behind the transfers with a tiled pipeline. Here a call is cut
 * into `chunks` column chunks so that the caller can overlap chunk c's
 * exchanges with chunk c + 1's kernels (on two streams ordered by events;
 * nothing in these kernels waits on another GPU).
 *
 * Chunk c of `chunks` takes, of every owner s's segment of len(s) groups,
 * the part [floor(c len(s) / chunks), floor((c + 1) len(s) / chunks)),
 * relative to the segment's first group (echo_query_chunk), so that every
 * owner receives 1/chunks of its segment in each chunk's all-to-all. The
 * partial last group (the last group of the last owner's segment) belongs to
 * the last chunk. Running chunks 0 .. chunks-1 of the three phases, each
 * chunk's exchanges between them, gives, bit for bit, the unchunked call.
 *
 *   echo_rank_quantize_chunk  phases 1, 2, 5 for this rank's non-owned groups
 *                             of the chunk: the send row's slots of every
 *                             owner's part
 *   all-to-all of the chunk   (caller) to owner s: send slots
 *                             [seg_begin(s) + first(s), + count(s)); owner s
 *                             puts what rank r sent at recv row r, slots
 *                             [first(s), first(s) + count(s))
 *   echo_rank_reduce_chunk    phases 1, 3, 5 for this rank's own part
 *   all-gather of the chunk   (caller) owner o's gsend slots
 *                             [first(o), first(o) + count(o)) to every rank's
 *                             gathered row o, same slots
 *   echo_rank_decode_chunk    phase 4 for every owner's part
 * (first/count from echo_query_chunk; codes are count * code_bytes bytes at
 * slot * code_bytes, parameter words count words at slot.)
 *
 *   chunk, chunks   0 <= chunk < chunks <= ECHO_MAX_CHUNKS; chunks = 1 is the
 *                   unchunked call (echo_rank_quantize & co. are these with
 *                   chunk 0 of 1)
 * Other arguments and errors as for the unchunked calls; ECHO_EINVAL for a
 * chunk out of range.
 */
#define ECHO_MAX_CHUNKS 4096

ECHO_API int echo_rank_quantize_chunk(const void* x, echo_state* st, int bits, float eta, float alpha_long,
                                      float alpha_short, float w, int chunk, int chunks, echo_stream_t stream);
ECHO_API int echo_rank_reduce_chunk(const void* x, void* out, echo_state* st, int bits, float eta,
                                    float alpha_long, float alpha_short, float w, int chunk, int chunks,
                                    echo_stream_t stream);
ECHO_API int echo_rank_decode_chunk(void* out, echo_state* st, int bits, int chunk, int chunks,
                                    echo_stream_t stream);

/*
 * Owner `owner`'s part of chunk `chunk` of `chunks`: *first = the part's
 * first group relative to the segment's first group, *count = its groups
 * (0 when the segment has fewer groups than chunks). Host-only, no device
 * call. ECHO_EINVAL for bad sizes, an owner outside [0, P) or a chunk out of
 * range.
 */
ECHO_API int echo_query_chunk(int64_t n, int P, int group, int owner, int chunk, int chunks, int64_t* first,
                              int64_t* count);

/*
 * ------------------------------------------------------------------------
 * The background-traffic study (the Echo abstract and the explainer's
 * results section "実測性能と精度": Echo's gain over a 16-bit all-reduce
 * grows with competing traffic). On one GPU the simulated transport is HBM,
 * so the competing traffic is an HBM copy on another stream.
 *
 * echo_bf16_allreduce_sim: the 16-bit baseline all-reduce simulated over P
 * virtual ranks like echo_allreduce_sim: every outputs[r] (n bf16) receives
 * bf16_rn of the binary32 sum of inputs[0..P-1] in rank order -- no
 * quantization, no state. Buffers as for echo_allreduce_sim (device, 16-byte
 * aligned; an output may be its own input). Asynchronous on `stream`.
 * ECHO_EINVAL on a bad size or pointer, ECHO_ECUDA on a launch error.
 */
ECHO_API int echo_bf16_allreduce_sim(const void* const* inputs, void* const* outputs, int64_t n, int P,
                                     echo_stream_t stream);

/*
 * echo_background_traffic: competing HBM traffic for duration_us
 * microseconds of wall-clock time: one single-warp CTA per SM copies src to
 * dst in 16 KB bulk copies through 32 KB of shared memory (bytes a multiple
 * of 16384, 16-byte aligned, not overlapping; the copy wraps around) during
 * the first duty_permille / 1000 of every period_us and sleeps for the rest. The kernel ends by itself when the duration has passed, whatever
 * else runs; it waits on nothing. When moved_dev is not NULL (8-byte aligned
 * device word) the bytes read and written are added to it. duty_permille 0
 * launches nothing.
 *   duty_permille 0 .. 1000, period_us 10 .. 10^6, duration_us 1 .. 6*10^7
 * Asynchronous on `stream` (give it a stream of its own so that it overlaps
 * the measured calls). ECHO_EINVAL on bad arguments, ECHO_ECUDA on a launch
 * error.
 */
ECHO_API int echo_background_traffic(const void* src, void* dst, size_t bytes, uint32_t duty_permille,
                                     uint32_t period_us, uint32_t duration_us, unsigned long long* moved_dev,
                                     echo_stream_t stream);

/* Release the host handle and the events echo_allreduce_sim_host created
 * for it (never the caller's device buffers). NULL is a no-op. */
ECHO_API int echo_free(echo_state* st);

/* Static string for a status code. */
ECHO_API const char* echo_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* ECHO_H */
