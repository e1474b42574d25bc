/*
 * vrar — virtual-rank all-reduce on one GPU (C ABI).
 *
 * P "virtual ranks" are P buffers in the memory of ONE CUDA device. A call
 * does every rank's reduce and exchange work on that device in a single
 * kernel launch: thread blocks act as the ranks and synchronise through flag
 * words and sequence-numbered 8-byte payload words in device memory. There is
 * no cross-GPU traffic and no collective library underneath.
 *
 * Sources for the operations (web pages; sections as printed on them):
 *  [CAR]   "fix(custom_all_reduce): use SYSTEM scope + ACQUIRE ordering for
 *          cross-device signal loads" (ROCm/aiter pull request 4786),
 *          "Summary" and "Root cause": start_sync / end_sync flag barriers
 *          polled with acquire loads, the 2-stage reduce-scatter + all-gather
 *          kernel, and its write mode, which streams the reduced slice into
 *          every rank's registered output and fences before end_sync.
 *  [NVRAR] "Understanding and Improving Communication Performance in
 *          Multi-node LLM Inference" (gist.science technical summary of
 *          arXiv 2511.09557), "Methodology" item 3 "Proposed Solution
 *          (NVRAR)": intra-node reduce-scatter, inter-node recursive doubling,
 *          intra-node all-gather; chunked non-blocking communication; data and
 *          flag fused into one 8-byte payload; sequence numbers in place of
 *          global barriers.
 *
 * Conventions for every call below
 *  - Buffers: rank_in[p] / rank_out[p] are DEVICE pointers on the CURRENT
 *    device (cudaGetDevice), each 16-byte aligned, each the start of a
 *    contiguous vector. The caller owns them. rank_in[] must not change, and
 *    rank_out[] must not be read, until the stream has passed the call.
 *  - The pointer arrays themselves are HOST arrays of P entries. They are
 *    copied into the kernel's parameters by value, so they may be freed or
 *    reused as soon as the call returns.
 *  - n is the number of ELEMENTS of the full per-rank vector.
 *  - Elements are bf16 (VRAR_BF16), IEEE binary16 (VRAR_FP16) or IEEE
 *    binary32 (VRAR_FP32). Sums are formed in binary32 with round-to-nearest-
 *    even adds and rounded to the element type with round-to-nearest-even
 *    (subnormals kept).
 *  - Out-of-place only: no output may overlap any input or another output.
 *  - 1 <= P <= VRAR_MAX_RANKS. n == 0 is a valid no-op.
 *  - The call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). It returns once the kernel is queued. Calls that run
 *    concurrently on different streams of one device are not supported: they
 *    share the device workspace.
 *  - The library owns a per-device workspace (flag words, payload slots, the
 *    sequence counter and a status word), allocated and zeroed on first use
 *    and grown when a larger call needs more. Growing allocates, which is not
 *    allowed while a stream is being captured into a CUDA graph: make one call
 *    of the largest shape (or call vrar_reserve) before capturing.
 *  - Settings (vrar_set_*) are read when a call is queued and become part of
 *    that launch; a call captured into a CUDA graph keeps the settings it was
 *    captured with.
 *  - Return value: VRAR_OK, or a negative VRAR_E* code. Argument errors are
 *    found on the host before anything is queued. A device wait that hits
 *    its time limit cannot be returned by the call that queued it: the kernel
 *    records VRAR_ETIMEDOUT in the status word, which vrar_query_status reads.
 *    No C++ exception crosses this interface.
 */
#ifndef VRAR_H
#define VRAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define VRAR_API __attribute__((visibility("default")))
#else
#define VRAR_API
#endif

#define VRAR_MAX_RANKS 32
#define VRAR_VERSION 1

/* Same type as cudaStream_t. */
typedef struct CUstream_st* vrar_stream_t;

typedef enum {
    VRAR_BF16 = 0,
    VRAR_FP32 = 1,
    VRAR_FP16 = 2   /* IEEE binary16 */
} vrar_dtype_t;

typedef enum {
    VRAR_ALGO_AUTO = 0,           /* per-size choice, see vrar_select_algo */
    VRAR_ALGO_ONESHOT = 1,        /* [CAR] 1-stage: every rank reads all P inputs */
    VRAR_ALGO_TWOSTAGE = 2,       /* [CAR] reduce-scatter, mid barrier, pull all-gather */
    VRAR_ALGO_TWOSTAGE_WRITE = 3, /* [CAR] write mode: owner streams its slice to all P outputs */
    VRAR_ALGO_RD = 4,             /* [NVRAR] recursive doubling with fused 8-byte payloads */
    VRAR_ALGO_HIER = 5            /* [NVRAR] group RS -> inter-group RD -> group AG */
} vrar_algo_t;

enum {
    VRAR_OK = 0,
    VRAR_EINVAL = -1,    /* bad argument: null/misaligned pointer, P or n out of range, overlap */
    VRAR_ENOTSUP = -2,   /* shape the algorithm does not define (RD: P not 2^k; HIER: L does not
                            divide P or P/L not 2^k) */
    VRAR_ENOMEM = -3,    /* workspace allocation failed */
    VRAR_ECUDA = -4,     /* a CUDA runtime call failed (no device, launch error, ...) */
    VRAR_ETIMEDOUT = -5, /* a device wait hit its time limit (reported by vrar_query_status) */
    VRAR_ETOOBIG = -6    /* request larger than the fixed scratch of vrar_allreduce_rd_noalloc */
};

/*
 * All-reduce. On return of the stream, every rank_out[p] (n elements) holds
 * the element-wise sum over ranks of rank_in[0..P-1] (n elements each); all P
 * outputs are bitwise identical. The order of the binary32 adds is fixed per
 * algorithm:
 *   ONESHOT, TWOSTAGE, TWOSTAGE_WRITE: ascending rank order from rank 0, one
 *     rounding to the element type at the end ([CAR] Summary; the order is
 *     this library's choice, the page fixes none).
 *   RD (P = 2^m): m steps; at step k rank p adds its partner p XOR 2^k's
 *     current partial to its own and rounds to the element type
 *     ([NVRAR] phase 2, "Fused Payloads"); with VRAR_WIRE_FP32 the partials
 *     stay fp32 and are rounded once at the end.
 *   HIER (P = G*L, rank r = g*L + l): ascending sum over the L ranks of group
 *     g, one rounding; then RD across the G groups; then copy to the group
 *     ([NVRAR] phases 1-3). L is set by vrar_set_group_size.
 *   AUTO: the algorithm vrar_select_algo returns, unless the environment
 *     variable VRAR_ALGO (oneshot|twostage|twostage_write|rd|hier) names one.
 */
VRAR_API int vrar_allreduce(const void* const rank_in[], void* const rank_out[], int P, size_t n,
                            vrar_dtype_t dtype, vrar_algo_t algo, vrar_stream_t stream);

/*
 * Reduce-scatter ([NVRAR] phase 1 over one group of P ranks). rank_in[p] has
 * n elements; rank_out[p] has n / P elements and receives elements
 * [p*n/P, (p+1)*n/P) of the ascending-rank sum. Requires n % P == 0.
 */
VRAR_API int vrar_reduce_scatter(const void* const rank_in[], void* const rank_out[], int P, size_t n,
                                 vrar_dtype_t dtype, vrar_stream_t stream);

/*
 * All-gather ([NVRAR] phase 3 over one group of P ranks). rank_in[p] has
 * n / P elements; rank_out[p] has n elements and receives
 * rank_in[0] | rank_in[1] | ... | rank_in[P-1] (exact copies). Requires
 * n % P == 0.
 */
VRAR_API int vrar_all_gather(const void* const rank_in[], void* const rank_out[], int P, size_t n,
                             vrar_dtype_t dtype, vrar_stream_t stream);

/*
 * The algorithm VRAR_ALGO_AUTO uses for (P, n, dtype) on the current device:
 * a table of per-size crossovers measured on a B200, in the spirit of the
 * size gates the sources show ([CAR] "Scope of impact": write mode only above
 * 4 MiB at 8 ranks). Never returns an algorithm that rejects the shape.
 * Returns a vrar_algo_t value, or VRAR_EINVAL.
 */
VRAR_API int vrar_select_algo(int P, size_t n, vrar_dtype_t dtype);

/*
 * Base name of the kernel that vrar_allreduce(.., P, n, dtype, algo, ..) would
 * launch under the current settings (AUTO resolved as vrar_allreduce resolves
 * it, the payload wire, the VRAR_WRITE_KERNEL override), e.g.
 * "k_twostage_write_async". Write mode has four kernels with one result:
 * "k_twostage_write" (plain: one item per thread and pass), "k_twostage_write_staged"
 * (bulk copies into shared memory by one producer lane), "k_twostage_write_async"
 * (per-thread async copies into shared memory), "k_twostage_write_batched" (two
 * items per thread and pass), chosen per shape from the same measured
 * table as vrar_select_algo (with fp8 payloads on, from a second measured table:
 * the algorithm AUTO runs stays the same). For profilers and benchmarks; the sources have
 * no counterpart. Returns a static string, or NULL for invalid arguments
 * (P outside 1..VRAR_MAX_RANKS, unknown dtype or algorithm). Launches nothing.
 */
VRAR_API const char* vrar_kernel_name(int P, size_t n, vrar_dtype_t dtype, vrar_algo_t algo);

/* Group size L used by VRAR_ALGO_HIER (default 8). Returns VRAR_OK or
 * VRAR_EINVAL (L < 1 or L > VRAR_MAX_RANKS). Process-wide setting. */
VRAR_API int vrar_set_group_size(int L);
VRAR_API int vrar_get_group_size(void);

/* Chunk count C of the recursive-doubling exchange (default 4): the vector is
 * cut into chunks and every thread keeps up to C payload pieces, one per chunk,
 * in flight per step ([NVRAR] "Chunked Non-blocking Communication"). A call
 * uses fewer than C when its grid has threads to spare for a short message.
 * VRAR_ALGO_RD on the element wire uses at most 2 (its kernel runs two CTAs
 * per SM with 64 registers per thread, measured faster than one CTA with more
 * pieces); VRAR_ALGO_HIER uses at most 2, and 1 up to 2 MiB per rank
 * (measured faster: its in-group phases keep L loads and stores per piece in
 * flight already); the fp32 wire at most 2; vrar_allreduce_rd_noalloc up to 8.
 * Results do not depend on C. Range 1..8. */
VRAR_API int vrar_set_rd_chunks(int C);
VRAR_API int vrar_get_rd_chunks(void);

/* What the fused payload words of RD and HIER carry ([NVRAR] "Fused
 * Payloads" does not say): VRAR_WIRE_ELEMENT (default) - the partial in the
 * element type, rounded at every step (2 bf16 / fp16 or 1 fp32 per word);
 * VRAR_WIRE_FP32 - the fp32 partial, rounded once at the end (1 float per
 * word: twice the words for bf16 / fp16, fewer roundings). For fp32 elements
 * the two are the same. The in-group sum of HIER is kept in fp32 too.
 * Process-wide setting; VRAR_EINVAL for other values. */
enum { VRAR_WIRE_ELEMENT = 0, VRAR_WIRE_FP32 = 1 };
VRAR_API int vrar_set_payload_wire(int wire);
VRAR_API int vrar_get_payload_wire(void);

/* fp8 payloads of the custom all-reduce: the ca_fp8_quant flag that the
 * ROCm/ATOM pull request 1681 page passes at the RowParallelLinear all-reduce
 * call site ("all_reduce(y, ca_fp8_quant=False)"). The page names the flag and
 * nothing more, so the scheme is this library's reading: with the setting on,
 * every value that passes from one rank to another in ONESHOT, TWOSTAGE and
 * TWOSTAGE_WRITE (and AUTO, which picks among them) travels as OCP FP8 E4M3
 * (4 exponent bits biased by 7, 3 fraction bits, subnormals kept, no
 * infinities, largest finite 448) with one binary32 scale per group of 8
 * elements (one 16-byte item of a bf16 / fp16 vector): s = amax / 448 (amax =
 * the group's largest magnitude; s = 1 when that gives 0), q = E4M3(x / s)
 * rounded to nearest even and saturated at 448, received as q * s (binary32
 * division and product, round to nearest even). ONESHOT passes every input
 * through it once (each rank's own input too, so all outputs agree):
 *   y = rnd_T(fp8(x_0) + fp8(x_1) + ... + fp8(x_{P-1}))   (binary32 adds, in order)
 * TWOSTAGE and TWOSTAGE_WRITE pass the inputs through it for the
 * reduce-scatter and the reduced binary32 slice again for the all-gather:
 *   y = rnd_T(fp8(fp8(x_0) + ... + fp8(x_{P-1})))
 * On one device nothing is stored in fp8: the kernels quantise and dequantise
 * in registers where a value would cross between ranks, so a call moves the
 * same bytes as without it. Inputs must be finite; a group whose binary32
 * sum overflows to infinity has an infinite scale in the 2-stage's second
 * quantisation and comes back as NaN. With the setting on, fp32 elements, RD
 * and HIER return VRAR_ENOTSUP. Default 0 (off). Process-wide setting, read
 * when a call is queued. */
VRAR_API int vrar_set_fp8_quant(int on);
VRAR_API int vrar_get_fp8_quant(void);

/* Whether ONESHOT / TWOSTAGE / TWOSTAGE_WRITE run the start and end flag
 * barriers of [CAR] (default 0 = no). Across devices they keep a rank from
 * reading a peer's buffer before the peer has entered the call, and from
 * returning while a peer still reads its buffer. Here every virtual rank runs
 * in one launch on one stream, so the launch boundaries already give both
 * guarantees and the barriers only add latency; 1 runs them anyway (same
 * results). The 2-stage mid barrier always runs: its all-gather reads other
 * ranks' partial results. */
VRAR_API int vrar_set_edge_sync(int on);
VRAR_API int vrar_get_edge_sync(void);

/* Upper bound on the CTAs one call launches (default 0 = the library's own
 * choice, at most what fits on the device at once: e.g. the plain write
 * kernel takes at most 128 on calls above 32 MiB, and recursive doubling
 * evens out its rounds; every call still gets at least one CTA per rank). A
 * budget leaves SMs to work running concurrently on other streams, e.g. the
 * partner micro-batch's GEMMs while this all-reduce runs on a communication
 * stream; the all-reduce is bound by memory bandwidth, which a fraction of
 * the SMs can already draw. With a budget of at most one CTA per SM the
 * write-mode and reduce-scatter kernels keep more bytes in flight per CTA
 * (deeper shared-memory stages). Results do not depend on the budget.
 * Process-wide setting. */
VRAR_API int vrar_set_max_ctas(int n);
VRAR_API int vrar_get_max_ctas(void);

/* Time limit of every device wait, in nanoseconds of %globaltimer
 * (default 2e9). Range 1e5 .. 6e10. */
VRAR_API int vrar_set_spin_timeout_ns(uint64_t ns);
VRAR_API uint64_t vrar_get_spin_timeout_ns(void);

/*
 * Wait for `stream`, then return and clear the device status words of the
 * current device: VRAR_OK, or VRAR_ETIMEDOUT if any wait of any call since
 * the last query ran out of time. This covers the calls that use the
 * library's workspace and those of vrar_allreduce_rd_noalloc, whose status
 * words live in its fixed array; both are cleared. If info is not NULL it
 * receives details of the first failure (the workspace's, if both failed):
 * info[0] = call sequence number, info[1] = phase (1 start, 2 mid, 3 end,
 * 4 payload, 5 shared-memory stage of the bulk-copy write kernel),
 * info[2] = waiting rank, info[3] = block. Allocates nothing.
 */
VRAR_API int vrar_query_status(vrar_stream_t stream, uint32_t info[4]);

/* Grow the current device's workspace now to at least `bytes` of payload
 * slots (so that later calls, e.g. under stream capture, need not allocate).
 * vrar_workspace_bytes returns the payload-slot bytes a call would need. */
VRAR_API int vrar_reserve(size_t bytes);
VRAR_API size_t vrar_workspace_bytes(int P, size_t n, vrar_dtype_t dtype, vrar_algo_t algo);

/* Free the current device's workspace (synchronises the device). The next
 * call allocates a fresh, zeroed one. */
VRAR_API int vrar_reset(void);

/*
 * Spin statistics of the cross-rank waits (flag barriers and payload polls),
 * after the temporary instrumentation described in [CAR] "Validation": off by
 * default; vrar_set_spin_stats(1) makes the following calls count, per wait,
 * how many polls it took (one extra warp-level reduction and a few atomics per
 * warp and wait). vrar_get_spin_stats waits for the device, then fills
 *   stats[0] waits counted        stats[1] polls in total
 *   stats[2] most polls in one wait
 *   stats[3] waits of 16384 polls or more
 *   stats[4] waits that hit the time limit (the "safety net")
 * for the current device, and clears the counters if `reset` is non-zero.
 * Returns VRAR_OK, VRAR_EINVAL (stats NULL) or VRAR_ECUDA.
 */
VRAR_API int vrar_set_spin_stats(int on);
VRAR_API int vrar_get_spin_stats(uint64_t stats[5], int reset);

/* Testing aid: ranks whose bit is set skip every flag post and payload send
 * of the following calls (until set back to 0), so that their peers' waits
 * run out of time and report VRAR_ETIMEDOUT instead of hanging. */
VRAR_API int vrar_debug_set_fault_mask(uint32_t mask);

/*
 * Allocation-free recursive-doubling all-reduce. The sources have no
 * counterpart of this call; it exists for callers that cannot let a library
 * allocate device memory: a serving process whose own allocator has already
 * claimed nearly all of the GPU's memory (a KV-cache pool, say) and must not
 * have memory taken behind its back, or code that must not block on the
 * device-wide synchronisation that cudaMalloc / cudaFree can imply.
 *
 * Same arguments, rules and results as vrar_allreduce(..., VRAR_ALGO_RD, ...)
 * (bit for bit), but it never allocates: its payload slots and control words
 * live in one fixed array of VRAR_NOALLOC_SCRATCH_BYTES compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits. It calls no cudaMalloc, no cudaFree and no allocating library routine.
 *  - Limit: P must be a power of two and
 *      256 + P * log2(P) * ceil(n / e) * 32 * w <= VRAR_NOALLOC_SCRATCH_BYTES
 *    (w = 2 with VRAR_WIRE_FP32 and 16-bit elements, else 1),
 *    e = 8 for bf16 / fp16, 4 for fp32 (P = 8, bf16: n <= 174,760). Larger
 *    requests return VRAR_ETOOBIG before anything is queued.
 *  - The first call on a device sets that device up: it looks up the array's
 *    device address (cudaGetSymbolAddress) and queues the array's zeroing
 *    (cudaMemsetAsync) on `stream`, ahead of the call's kernel. Make that
 *    first call before any stream capture.
 *  - All calls on a device share the one array, and it keeps the last call's
 *    contents; nothing has to be cleared between calls, because every word a
 *    call waits for carries that call's sequence number. Calls that overlap on
 *    the GPU (on different streams, or from several host threads) race on the
 *    array and give wrong results: keep them ordered on one stream.
 *  - The CUDA driver can reserve device memory behind any kernel launch, which
 *    this call cannot prevent: with lazy module loading (the default since
 *    CUDA 12.2) it loads a kernel's code the first time that kernel is used,
 *    and it reserves local memory for the whole device the first time it runs
 *    a kernel that needs local memory. This call picks, among the kernel
 *    variants that suit the request, one that uses no local memory (asked of
 *    the runtime with cudaFuncGetAttributes); with CUDA_MODULE_LOADING=EAGER
 *    in the environment all of the library's code is loaded when the library
 *    first calls the CUDA runtime, and a call then changes the device's free
 *    memory by nothing.
 *  - Device waits are bounded as in every other call (vrar_set_spin_timeout_ns)
 *    and honour vrar_debug_set_fault_mask. A wait that runs out of time
 *    records VRAR_ETIMEDOUT in the array's status word, and the outputs of the
 *    items whose waits gave up are left unwritten; vrar_query_status reports
 *    and clears it. Spin statistics are not collected on this path.
 */
#define VRAR_NOALLOC_SCRATCH_BYTES (16u << 20)
VRAR_API int vrar_allreduce_rd_noalloc(const void* const rank_in[], void* const rank_out[], int P, size_t n,
                                       vrar_dtype_t dtype, vrar_stream_t stream);

/* Static description of a return code. */
VRAR_API const char* vrar_strerror(int code);

VRAR_API int vrar_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VRAR_H */
