/*
 * mpe.h -- mixed-precision MoE experts served from paged 3/4/8-bit weights.
 *
 * C ABI of libmpe.so. Plain pointers and sizes only; every array argument
 * states whether it lives in host or device memory. All device work runs in
 * the library's CUDA kernels (sm_100a) on the context's stream.
 *
 * The operations follow the PagedWeight method ("PagedWeight: Efficient MoE
 * LLM Serving with Dynamic Quality-Aware Weight Quantization", llmdb.app
 * summary page):
 *   - allocate precision per expert under a weight budget B
 *     ("Quality-Aware Quantization": min sum_e p_e L(b_e) s.t. sum_e b_e W_e <= B);
 *   - quantize each expert with one absmax scale and store it in pages of its
 *     bit width, reached through a page table keyed by expert ID
 *     ("Implementation Details": Q(w) = round(w/s) s, s = max|w|/(2^(b-1)-1);
 *     memory management via a page table; "Dynamic Paging": pages of 8/4/3 bits);
 *   - run the routed expert FFN straight from those pages, dequantizing on the
 *     fly ("Dynamic Paging": the router picks experts, their pages are fetched
 *     and dequantized on the fly);
 *   - re-quantize when the budget changes with KV-cache occupancy ("Implementation
 *     Details": the scheduler adjusts page sizes with KV-cache occupancy).
 *
 * Error behaviour: every int-returning call returns MPE_OK (0) or a negative
 * MPE_ERR_* code; a human-readable message is kept per context (mpe_last_error)
 * or per thread for calls without a context. No call exits, throws or traps.
 * Device-side faults that kernels detect (an out-of-range expert id, NaN/Inf
 * in a master, a bounded wait that ran out) set bits of a sticky status word
 * read by mpe_get_status; kernels skip the offending work instead of faulting.
 *
 * Thread safety: a context may be used by one host thread at a time.
 */
#ifndef MPE_H
#define MPE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------ */
#define MPE_OK               0
#define MPE_ERR_INVALID     -1  /* bad argument: null pointer, size or alignment      */
#define MPE_ERR_INFEASIBLE  -2  /* B < 3 * sum_e W_e                                  */
#define MPE_ERR_STATE_CAP   -3  /* budget needs more allocation states than the cap   */
#define MPE_ERR_POOL        -4  /* page pool exhausted; nothing was changed           */
#define MPE_ERR_CUDA        -5  /* a CUDA runtime call failed (message has details)   */
#define MPE_ERR_ORDER       -6  /* call out of order, e.g. moe_ffn before quantize    */
#define MPE_ERR_DEVICE      -7  /* a kernel reported a problem: see mpe_get_status    */

/* ---- sticky device status bits (mpe_get_status) ------------------------ */
#define MPE_STATUS_BAD_EXPERT_ID   0x1u  /* an id outside [0, E): that slot was dropped */
#define MPE_STATUS_NONFINITE       0x2u  /* a master holds NaN/Inf: expert not encoded  */
#define MPE_STATUS_WAIT_TIMEOUT    0x4u  /* a bounded device wait gave up               */
#define MPE_STATUS_ALLOC_INFEASIBLE 0x8u /* allocator kernel: B < 3 * sum W             */
#define MPE_STATUS_ALLOC_STATE_CAP 0x10u /* allocator kernel: too many states           */

/* ---- limits ------------------------------------------------------------- */
#define MPE_MAX_EXPERTS        1024  /* E                                               */
#define MPE_ALLOC_STATE_CAP    65536 /* allocator DP states (budget units + 1)          */
#define MPE_DEFAULT_PAGE_BYTES 65536
#define MPE_MAX_COMP_CHANNELS  256   /* salient channels compensated per input row    */
#define MPE_MAX_ASSIGNMENTS    (1 << 24) /* T*k per forward / route call               */

/* ---- forward-pass path selection --------------------------------------- */
#define MPE_PATH_AUTO    0   /* decode kernels for small token counts, prefill above */
#define MPE_PATH_DECODE  1   /* force the grouped GEMV (mma.sync) path              */
#define MPE_PATH_PREFILL 2   /* force the tcgen05 grouped GEMM path                  */

/*
 * Layer shape and resources. E experts, each a SwiGLU FFN with gate W1 [F x H],
 * up W3 [F x H] and down W2 [H x F] (row = output feature, K contiguous).
 * H and F must be multiples of 128.
 */
typedef struct mpe_config {
    int32_t  E;            /* experts, 1 .. MPE_MAX_EXPERTS                                 */
    int32_t  H;            /* hidden size, multiple of 128                                  */
    int32_t  F;            /* expert FFN size, multiple of 128                              */
    uint32_t page_bytes;   /* physical page size; 0 = 65536; multiple of 4096, >= 4096      */
    uint32_t pool_pages;   /* pages in the pool; 0 = enough for every expert at 8 bits      */
    int32_t  device;       /* CUDA device ordinal; -1 = the current device                  */
    int32_t  path;         /* MPE_PATH_*                                                    */
    int32_t  reserved;
    void*    stream;       /* cudaStream_t for all work; NULL = the legacy default stream   */
} mpe_config;

/* One page-table entry: expert e's pages are page_idx[first .. first+n_pages). */
typedef struct mpe_pte {
    uint8_t  bits;         /* 3, 4 or 8; 0 = not quantized yet   */
    uint8_t  pad[3];
    float    scale;        /* s_e = RN_f32(max|w| / (2^(b-1)-1)) */
    uint32_t first;        /* index into the page-index array    */
    uint32_t n_pages;      /* pages held by the expert           */
} mpe_pte;

typedef struct mpe_ctx mpe_ctx;

/*
 * mpe_create -- make a context: device page pool, page table, caches and
 * scratch, all owned by the library. *out receives the context (host pointer).
 * Returns MPE_ERR_INVALID for a bad shape, MPE_ERR_CUDA if allocation fails.
 */
int mpe_create(mpe_ctx** out, const mpe_config* cfg);

/* mpe_destroy -- synchronise the context's stream and free everything it owns. */
void mpe_destroy(mpe_ctx* ctx);

/* mpe_set_stream -- run later work on `stream` (a cudaStream_t; NULL = default). */
int mpe_set_stream(mpe_ctx* ctx, void* stream);

/* mpe_set_path -- choose the forward-pass path (MPE_PATH_*). */
int mpe_set_path(mpe_ctx* ctx, int32_t path);

/*
 * mpe_allocate_bits -- PagedWeight's allocation problem
 * ("Quality-Aware Quantization"): choose b_e in {3,4,8} minimising
 * sum_e p_e L(b_e) subject to sum_e b_e W_e <= B_bits, L(b) = 1/(2^(b-1)-1)^2,
 * solved exactly by a dynamic program in one device kernel on the current
 * device. Ties keep the lower width and the lower budget.
 *   p        host, float64[E], importances
 *   W        host, uint64[E], weight elements per expert (> 0)
 *   E        1 .. MPE_MAX_EXPERTS
 *   B_bits   budget in bits of codes
 *   bits_out host, uint8[E], receives b_e
 * Synchronous. MPE_ERR_INFEASIBLE if B_bits < 3 sum W; MPE_ERR_STATE_CAP if
 * (B_bits - 3 sum W) / gcd(W) + 1 exceeds MPE_ALLOC_STATE_CAP.
 */
int mpe_allocate_bits(const double* p, const uint64_t* W, int32_t E, uint64_t B_bits,
                      uint8_t* bits_out);

/*
 * mpe_allocate_bits_proportional -- the page's simplified allocator
 * ("Code Illustration", compute_budgeted_precision): expert e's share of the
 * budget, B_bits p_e / sum p, in bits per weight (share / W_e) rounded up to
 * the next width (3 if <= 3, 4 if <= 4, else 8); then, since rounding up can
 * exceed the budget, experts in ascending (p_e, e) are downgraded one width at
 * a time (8 -> 4 -> 3) until sum b_e W_e <= B_bits (the repair is this
 * library's addition). float64 throughout, sum p in ascending e; one device
 * kernel on the current device. Same arguments as mpe_allocate_bits.
 * Synchronous. MPE_ERR_INFEASIBLE if B_bits < 3 sum W.
 */
int mpe_allocate_bits_proportional(const double* p, const uint64_t* W, int32_t E,
                                   uint64_t B_bits, uint8_t* bits_out);

/*
 * mpe_allocate_bits_table -- the same exact program with a loss per expert
 * and width: minimise sum_e p_e loss[e][b_e] subject to sum_e b_e W_e <= B_bits
 * (PagedWeight, "Quality-Aware Quantization": L(b) is a loss such as the mean
 * squared error, and experts differ in sensitivity). Each cost is one float64
 * multiply p_e * loss[e][b]; ties keep the lower width and the lower budget.
 * Unlike mpe_allocate_bits, a budget of 8 sum W or more is solved too (each
 * expert then takes its least cost, which need not be 8 bits).
 *   loss     host, float64[E][3], row e = (loss at 3, 4, 8 bits), finite, >= 0;
 *            e.g. the output of mpe_measure_loss
 *   other arguments as for mpe_allocate_bits
 * Synchronous. Same errors as mpe_allocate_bits.
 */
int mpe_allocate_bits_table(const double* p, const double* loss, const uint64_t* W, int32_t E,
                            uint64_t B_bits, uint8_t* bits_out);

/* width rules mpe_repage can use (mpe_set_allocator) */
#define MPE_ALLOCATOR_EXACT        0  /* mpe_allocate_bits (default)            */
#define MPE_ALLOCATOR_PROPORTIONAL 1  /* mpe_allocate_bits_proportional         */
#define MPE_ALLOCATOR_MEASURED     2  /* mpe_allocate_bits_table with the
                                         context's mpe_measure_loss values      */

/* mpe_set_allocator -- choose the width rule of later mpe_repage calls
 * (MPE_ALLOCATOR_MEASURED measures the losses on first use). */
int mpe_set_allocator(mpe_ctx* ctx, int32_t allocator);

/*
 * mpe_quantize_experts -- quantize every expert at the given widths
 * ("Implementation Details", quantization scheme): per-expert absmax m_e
 * (cached: the master must not change while the context lives), scale
 * s_e = RN_f32(m_e / (2^(b-1)-1)), codes k = round-half-even(w / s_e) clamped
 * to +-(2^(b-1)-1), stored offset-binary in chunks of 16 rows x 128 codes,
 * placed in the pool's pages (lowest free page first, experts ascending) and
 * recorded in the page table.
 *   master_f16 host array of E device pointers; expert e's fp16 master is
 *              W1 [F x H] | W3 [F x H] | W2 [H x F], row-major, contiguous,
 *              16-byte aligned. Borrowed: it must outlive the context
 *              (mpe_repage re-reads it).
 *   bits       host, uint8[E], each 3, 4 or 8.
 * Asynchronous on the context stream (the page table is uploaded from
 * context-owned host memory). A NaN/Inf master sets MPE_STATUS_NONFINITE.
 * MPE_ERR_POOL if the pool is too small (nothing changes).
 */
int mpe_quantize_experts(mpe_ctx* ctx, const void* const* master_f16, const uint8_t* bits);

/*
 * mpe_measure_loss -- the measured quantization error of every expert at
 * every width: loss[e][i] = (1/n) sum (w - k s_b)^2 over expert e's n = 3 H F
 * fp16 master weights, with that width's own scale s_b = RN_f32(m_e / q_b)
 * and codes k = round-half-even(w / s_b), for b = 3, 4, 8 (i = 0, 1, 2). The
 * sum of squares is exact (integer arithmetic on the device), rounded once to
 * float64, then divided by n in float64. A zero expert gives 0, a non-finite
 * master NaN. Measured once per context (the master is immutable) and kept
 * for MPE_ALLOCATOR_MEASURED.
 *   loss_host  host, float64[E][3]
 * Synchronous. MPE_ERR_ORDER before mpe_quantize_experts.
 */
int mpe_measure_loss(mpe_ctx* ctx, double* loss_host);

/* where mpe_set_compensation keeps its residual store */
#define MPE_STORE_DEVICE 0  /* device memory                                        */
#define MPE_STORE_HOST   1  /* mapped pinned host memory, read by the kernels over
                               the bus (the CPU-side residuals of the paper)        */

/*
 * mpe_set_compensation -- dynamic error compensation of salient input
 * channels on the streaming path (DecDEC summary, 3.1-3.2: each quantized
 * linear W^ x becomes (W^ + R (.) M) x with R = W - W^ and M keeping the input
 * channels of largest |x|). With n_channels > 0 every later mpe_moe_ffn keeps,
 * per input row (a token's x for gate and up, a routed position's h for
 * down), its n_channels channels of largest |x| (ties to the lower index; all
 * of them when the row is shorter) and adds R[:, c] x_c for those channels,
 * so their weights are exactly the fp16 master values. R is recomputed from a
 * transposed copy of the masters (the residual store, 2 bytes per weight)
 * and each expert's current scale.
 *   n_channels  0 (off: the store is released) .. MPE_MAX_COMP_CHANNELS
 *   store       MPE_STORE_DEVICE or MPE_STORE_HOST
 * Synchronous (builds the store from the borrowed masters; mpe_quantize_experts
 * rebuilds it). While on, MPE_PATH_AUTO takes the streaming path and
 * mpe_moe_ffn fails with MPE_ERR_INVALID under MPE_PATH_PREFILL.
 * MPE_ERR_ORDER before mpe_quantize_experts; MPE_ERR_CUDA if the store cannot
 * be allocated (compensation stays off).
 */
int mpe_set_compensation(mpe_ctx* ctx, int32_t n_channels, int32_t store);

/*
 * mpe_get_kept_channels -- the channels the last compensated mpe_moe_ffn kept:
 * which = 0: per token, x's channels (gate and up), int32 [T][n];
 * which = 1: per route position, h's channels (down), int32 [T k][n]
 * (route positions: the experts' buckets in expert order, the slots of an
 * expert in assignment order t k + j). A row holds min(n, row length)
 * ascending entries; n is the compensation's n_channels.
 *   idx_host  host, int32, at least cap entries
 * Synchronous. MPE_ERR_ORDER if compensation is off or nothing ran yet;
 * MPE_ERR_INVALID if cap is too small.
 */
int mpe_get_kept_channels(mpe_ctx* ctx, int32_t which, int32_t* idx_host, size_t cap);

/*
 * mpe_select_salient -- the channel choice of the compensation on its own:
 * for each of n_rows rows of n_cols bf16 values, the n channels of largest
 * magnitude (ties to the lower index), ascending; every channel when
 * n >= n_cols. Allocates nothing; asynchronous on `stream`.
 *   rows_bf16  device, bf16 [n_rows][n_cols], row-major
 *   idx_out    device, int32 [n_rows][n]; row r's first min(n, n_cols)
 *              entries are written
 *   n          1 .. MPE_MAX_COMP_CHANNELS
 *   stream     cudaStream_t (NULL: the default stream)
 */
int mpe_select_salient(const void* rows_bf16, int32_t n_rows, int32_t n_cols, int32_t n,
                       int32_t* idx_out, void* stream);

/*
 * mpe_repage -- budget change with KV-cache occupancy ("Implementation
 * Details"; 0to1log digest: lower precision as the KV cache grows, raise it
 * as it shrinks): re-run the context's width rule (mpe_allocate_bits, or
 * mpe_allocate_bits_proportional / the measured-loss program after
 * mpe_set_allocator) with B_bits and
 * importances p (host float64[E]), release the pages of experts whose width
 * changed, give
 * them new pages and re-encode only those experts from the fp16 master with
 * the cached absmax. *n_changed_out (host, may be NULL) receives the count.
 * The width rule runs on a context-internal stream of the highest priority,
 * beside the work already queued on the context stream (it reads only p and
 * the expert sizes), and the call waits for it (the new widths decide the
 * page moves); the page-table upload, the scales and the encode are queued
 * on the context stream after the work already there, and the call returns
 * without waiting for them. MPE_ERR_POOL leaves widths, pages and codes
 * unchanged.
 */
int mpe_repage(mpe_ctx* ctx, uint64_t B_bits, const double* p, int32_t* n_changed_out);

/*
 * mpe_repage_async -- the same budget change overlapped with serving: the new
 * widths come from the context's width rule as in mpe_repage, but the changed
 * experts' old pages stay in use -- mpe_moe_ffn keeps reading the current page
 * table -- while the new page table is prepared and the changed experts are
 * re-encoded into pages that are free now (lowest first, ascending e) on an
 * internal stream of the context. The switch happens at mpe_repage_commit,
 * which also returns the old pages to the pool.
 *   B_bits, p, n_changed_out   as for mpe_repage
 * Synchronises the internal stream once (the widths); the encode is
 * asynchronous. The pool needs free pages for the changed experts' new pages
 * beside the old ones: MPE_ERR_POOL (nothing changed) otherwise.
 * MPE_ERR_ORDER if a previous overlapped repage is not committed. Until the
 * commit, mpe_get_bits reports the new widths; mpe_quantize_experts,
 * mpe_repage, mpe_get_page_table, mpe_get_scales and mpe_read_expert_packed
 * commit first (waiting on the device, not the host).
 */
int mpe_repage_async(mpe_ctx* ctx, uint64_t B_bits, const double* p, int32_t* n_changed_out);

/*
 * mpe_repage_commit -- switch later work to the page table of the pending
 * overlapped repage. wait = 0: only if its device work has finished
 * (*committed = 0 otherwise, nothing changes); wait != 0: always -- later work
 * on the context stream is ordered after that device work (the host does not
 * block). *committed (host, may be NULL) = 1 when no repage is pending.
 */
int mpe_repage_commit(mpe_ctx* ctx, int32_t wait, int32_t* committed);

/*
 * mpe_moe_ffn -- the routed expert SwiGLU FFN run from the pages ("Dynamic
 * Paging"): bucket the T*k (token, slot) assignments by expert, then for each
 * expert with tokens, stream its pages through the page table, unpack and
 * dequantize in registers, and compute g = s W1 x, v = s W3 x,
 * h = silu(g) v (rounded to bf16), y = s W2 h with fp32 accumulation;
 * out[t] = bf16(sum_j w[t,j] y_{t,j}), summed in fp32.
 *   x    device, bf16 [T x H], 16-byte aligned rows
 *   T    tokens (>= 0)
 *   ids  device, int32 [T x k]; ids outside [0,E) are dropped and set
 *        MPE_STATUS_BAD_EXPERT_ID
 *   w    device, float32 [T x k] top-k weights
 *   k    1 .. 32
 *   out  device, bf16 [T x H]
 * Two contraction paths compute the same values: a streaming one (packed
 * pages read once per work group of up to 16 tokens, warp-level MMA) and a
 * tensor-core one (tcgen05 MMA over work groups of up to 192 tokens, the
 * weights dequantized to bf16 straight into tensor memory as the MMA's A
 * operand, the tokens brought into shared memory by TMA and shared by two
 * weight tiles). MPE_PATH_AUTO takes the tensor-core path when T*k >= 32 E.
 * T*k above MPE_MAX_ASSIGNMENTS: MPE_ERR_INVALID.
 * Asynchronous on the context stream; scratch grows on demand (that call
 * synchronises).
 */
int mpe_moe_ffn(mpe_ctx* ctx, const void* x, int32_t T, const int32_t* ids, const float* w,
                int32_t k, void* out);

/*
 * mpe_moe_ffn_host -- mpe_moe_ffn with HOST buffers (preferably pinned):
 * copies x, ids and w to context-owned device staging, runs the layer and
 * copies out back, then synchronises. Same shapes as mpe_moe_ffn. It runs on
 * a context-internal stream ordered after the work queued on the context
 * stream; when the same (T, k) repeats with no reallocation, path or
 * compensation change in between, its kernels replay as one CUDA graph.
 */
int mpe_moe_ffn_host(mpe_ctx* ctx, const void* x_host, int32_t T, const int32_t* ids_host,
                     const float* w_host, int32_t k, void* out_host);

/*
 * mpe_moe_ffn_host_async -- mpe_moe_ffn_host without the final wait: queues
 * the copies in, the layer and the copy out, and returns a ticket in *ticket.
 * The copies in and the copies out run on two context-internal streams and
 * the layer on the internal compute stream, through two device staging slots
 * taken in turn, so one call's copies overlap the neighbouring calls' layers.
 * Any number of calls may be queued; each waits on the device for whatever it
 * must not overtake (its slot's previous call, the work already queued on the
 * context stream), and later work on the context stream waits for it. The
 * call's host buffers are the library's until mpe_host_wait(ticket) returns:
 * x_host, ids_host and w_host must stay unchanged and out_host unread until
 * then (pinned memory, or the copies are synchronous). T = 0 queues nothing
 * and returns the ticket UINT64_MAX. Errors as for mpe_moe_ffn_host.
 */
int mpe_moe_ffn_host_async(mpe_ctx* ctx, const void* x_host, int32_t T, const int32_t* ids_host,
                           const float* w_host, int32_t k, void* out_host, uint64_t* ticket);

/*
 * mpe_host_wait -- blocks until the call with this ticket has finished,
 * its output copied to out_host (it may also wait for later calls queued
 * on the same staging slot). UINT64_MAX returns at once. MPE_ERR_INVALID for
 * a ticket not yet issued; MPE_ERR_CUDA if the device reported an error.
 */
int mpe_host_wait(mpe_ctx* ctx, uint64_t ticket);

/*
 * mpe_route -- the bucketing step alone (for inspection): perm = the
 * assignments a = t*k + j sorted stably by expert id, offsets[E+1] = exclusive
 * prefix sums of the per-expert counts, inv[a] = position of a in perm (-1 for
 * dropped ids). Device pointers: ids int32 [T*k], perm int32 [T*k],
 * offsets int32 [E+1], inv int32 [T*k]. Asynchronous. T*k above
 * MPE_MAX_ASSIGNMENTS: MPE_ERR_INVALID.
 */
int mpe_route(mpe_ctx* ctx, const int32_t* ids, int32_t T, int32_t k, int32_t* perm,
              int32_t* offsets, int32_t* inv);

/*
 * mpe_route_noalloc -- the same bucketing as mpe_route (perm, offsets, inv;
 * identical results) for callers that cannot allocate device memory when they
 * route: a serving engine that fixes its GPU memory plan up front, or code
 * running while another component owns the allocator. It needs no context and
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine);
 * its working memory is one file-scope device array that every GPU loading the
 * library keeps until the process exits. The pages have no counterpart for
 * this call: it is an engineering variant of mpe_route.
 *   ids      device, int32 [T*k]; ids outside [0,E) are dropped (inv = -1)
 *   T, k     tokens and slots per token, 1 <= k <= 32; T*k <= 65536
 *   E        experts, 1 .. MPE_MAX_EXPERTS
 *   perm     device, int32 [T*k]; offsets device, int32 [E+1];
 *   inv      device, int32 [T*k]
 *   stream   cudaStream_t (NULL = the legacy default stream)
 * Each call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, which allocates nothing) and sets the kernels'
 * shared-memory limit there, so a device reset between calls is harmless; the
 * first call on a device also loads the library's kernels onto it, so make
 * that first call before any stream capture. All calls on a device share the
 * array: calls that overlap on the GPU (different streams, no ordering
 * between them) race and must not be issued. Asynchronous. With T*k = 0 only
 * offsets is written (all zero) and ids, perm, inv may be NULL.
 * MPE_ERR_INVALID (message in mpe_last_error_global) for a null pointer, a
 * bad E/T/k or T*k above 65536. MPE_ERR_CUDA if a CUDA error from earlier
 * work is pending on the calling thread when the call starts (it is left
 * pending, and the message says it came from earlier work), or if one of the
 * call's own launches fails (the message names the kernel).
 */
int mpe_route_noalloc(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t* perm,
                      int32_t* offsets, int32_t* inv, void* stream);

/*
 * mpe_get_page_table -- copy the page table to host: pte_host mpe_pte[E] and
 * page_idx_host uint32[cap] (the compact page-index array; its length is the
 * sum of n_pages). Either pointer may be NULL. Synchronous.
 * MPE_ERR_INVALID if cap is smaller than the array.
 */
int mpe_get_page_table(mpe_ctx* ctx, mpe_pte* pte_host, uint32_t* page_idx_host, size_t cap);

/*
 * mpe_expert_stream_bytes -- bytes of expert e's chunk stream at its current
 * width (b * W_e / 8); 0 if not quantized.
 */
size_t mpe_expert_stream_bytes(mpe_ctx* ctx, int32_t e);

/*
 * mpe_read_expert_packed -- gather expert e's chunk stream out of its pages
 * into host_dst (bytes >= the stream size), in stream order: W1 and W3 chunks
 * alternating (chunk 2c is W1's chunk c, 2c+1 W3's), then W2's chunks with
 * row tiles 2v and 2v+1 alternating by block column.
 * Synchronous.
 */
int mpe_read_expert_packed(mpe_ctx* ctx, int32_t e, void* host_dst, size_t bytes);

/*
 * mpe_get_scales -- host float32[E] scales and float32[E] absmax values
 * (either may be NULL). Synchronous.
 */
int mpe_get_scales(mpe_ctx* ctx, float* scale_host, float* absmax_host);

/* mpe_get_bits -- host uint8[E] current widths (0 = not quantized). */
int mpe_get_bits(mpe_ctx* ctx, uint8_t* bits_host);

/*
 * mpe_get_status -- synchronise the stream and return the sticky device
 * status word (MPE_STATUS_* bits) in *status_out; clear it if `clear` != 0.
 */
int mpe_get_status(mpe_ctx* ctx, uint32_t* status_out, int32_t clear);

/* mpe_last_error -- message for the context's last failure ("" if none). */
const char* mpe_last_error(mpe_ctx* ctx);

/* mpe_last_error_global -- message for the calling thread's last failure of a
 * context-free call (mpe_allocate_bits, mpe_create). */
const char* mpe_last_error_global(void);

/*
 * mpe_profile_enable -- when enable != 0, mpe_moe_ffn records a CUDA event
 * pair around each of its kernels (on the context stream) so their device
 * times can be read back; 0 stops recording. Recording costs one event
 * record per kernel boundary.
 */
int mpe_profile_enable(mpe_ctx* ctx, int32_t enable);

/*
 * mpe_profile_read -- synchronise and sum the recorded kernel times per slot
 * (0 route, 1 gate/up, 2 SwiGLU reduce, 3 down, 4 combine -- the streaming
 * path; 5 gate/up, 6 down, 7 token permute -- the tensor-core path; route
 * and combine are shared; 8 salient-channel selection, 9 compensation --
 * with mpe_set_compensation): ms_host
 * double[n_slots] milliseconds, launches_host int64[n_slots] counts (either
 * may be NULL). reset != 0 clears the records.
 */
int mpe_profile_read(mpe_ctx* ctx, double* ms_host, int64_t* launches_host, int32_t n_slots,
                     int32_t reset);

/*
 * mpe_selftest_wait -- exercises the failure path of the bounded device
 * waits without a fault: a kernel waits on a shared-memory barrier that
 * nothing completes, gives up after limit_ns (1 .. 1e9) and sets
 * MPE_STATUS_WAIT_TIMEOUT in the status word (read it with mpe_get_status);
 * nothing is left in flight and the context stays usable. Synchronous.
 */
int mpe_selftest_wait(mpe_ctx* ctx, uint64_t limit_ns);

/* mpe_kernel_launches -- how many kernels this context has launched so far. */
uint64_t mpe_kernel_launches(mpe_ctx* ctx);

/* mpe_version -- library version, e.g. 100 for 0.1.0. */
int32_t mpe_version(void);

/* ------------------------------------------------------------------------
 * Prefix-compatible variant (a separate store). A nested grid -- 2^b uniform
 * bins over [-m, m], m = max |w| of the expert, values at the bin centres --
 * makes every width's code the top bits of the 8-bit code:
 *   u8 = clamp(floor(128 w / m) + 128, 0, 255), u_b = u8 >> (8 - b),
 *   w^_b = (m / 2^b)(2 u_b + 1 - 2^b).
 * The codes are stored in layers, each in its own pages: A = u8 >> 5
 * (3 bits), B = bit 4 of u8, C = u8 & 15; a b-bit expert holds A, A B or
 * A B C. A layer is a chunk stream in the main format's layout at the layer's
 * width: chunks of 16 rows x 128 codes in the expert stream's order (W1 and
 * W3 alternating, then W2 by tile pairs), a row's codes as four quarters of
 * 32 -- A in the 3-bit quarter layout, C in the 4-bit one, B in a 1-bit
 * quarter (code c'_i at bit 16 (i & 1) + (i >> 1) of one word); a page holds
 * whole chunks (256 x layer bits bytes each). Lowering a width frees
 * the dropped layers' pages and encodes nothing; raising it adds pages for
 * the new layers and encodes only those (one read of the master). Placement
 * takes the lowest free pages, experts ascending, layers A, B, C; a repage
 * frees first (ascending e) and allocates after (ascending e).
 * ------------------------------------------------------------------------ */
typedef struct mpe_prefix mpe_prefix;

/* mpe_prefix_create -- a store for cfg->E experts of cfg->H x cfg->F (path is
 * ignored; pool_pages 0 = every expert at 8 bits). *out is owned by the
 * caller (mpe_prefix_destroy). MPE_ERR_INVALID / MPE_ERR_CUDA. */
int mpe_prefix_create(mpe_prefix** out, const mpe_config* cfg);
void mpe_prefix_destroy(mpe_prefix* store);
const char* mpe_prefix_last_error(mpe_prefix* store);

/* mpe_prefix_quantize -- m_e and all stored layers of every expert at the
 * given widths. master_f16: host array of E device pointers as for
 * mpe_quantize_experts (borrowed; repage re-reads it); bits: host uint8[E],
 * each 3, 4 or 8. Synchronous. MPE_ERR_POOL if the pool is too small. */
int mpe_prefix_quantize(mpe_prefix* store, const void* const* master_f16, const uint8_t* bits);

/* mpe_prefix_repage -- new widths (host uint8[E]); *bytes_moved_out (may be
 * NULL) receives the bytes the change moved: per expert that gains layers,
 * one read of its master (2 bytes a weight) plus the added layers written;
 * experts that only lose layers move nothing. Synchronous; waits for work
 * already queued (it may read the dropped pages). MPE_ERR_POOL leaves
 * everything unchanged. */
int mpe_prefix_repage(mpe_prefix* store, const uint8_t* new_bits, uint64_t* bytes_moved_out);

/* mpe_prefix_moe_ffn -- the routed SwiGLU layer from the layered store, same
 * arguments, checks and result layout as mpe_moe_ffn (x, ids, w, out device,
 * x and out 16-byte aligned, k <= 32, T k <= MPE_MAX_ASSIGNMENTS; ids outside
 * [0, E) contribute nothing). The expert is dequantized as w^_b above, in
 * registers inside the streaming path's kernels, which read the stored
 * layers of each chunk side by side. Asynchronous on the store's stream. */
int mpe_prefix_moe_ffn(mpe_prefix* store, const void* x_bf16, int32_t T, const int32_t* ids,
                       const float* w, int32_t k, void* out_bf16);

/* mpe_prefix_read_layer -- layer (0 A, 1 B, 2 C) of expert e in stream order
 * into host_dst (3 H F / 2048 chunks of 768 / 256 / 1024 bytes), read
 * through the device page table. Synchronous. MPE_ERR_INVALID if the layer
 * is not stored or the buffer is short. */
int mpe_prefix_read_layer(mpe_prefix* store, int32_t e, int32_t layer, void* host_dst,
                          size_t bytes);

/* mpe_prefix_get_absmax -- m_e of every expert (host float[E]). */
int mpe_prefix_get_absmax(mpe_prefix* store, float* m_host);

#ifdef __cplusplus
}
#endif

#endif /* MPE_H */
