/*
 * xs.h -- C ABI of libxs.so: non-causal DiT self-attention fused, tile by tile, with the
 * Ulysses post-attention All-to-All, for NVIDIA B200 (sm_100a).
 *
 * The operation (page "X-Stage: An Overlooked Pipeline Stage for Communication-Computation
 * Overlap in DiT Inference": abstract, and the explainer's "Technisches Resuemee" ->
 * "Zentrale Beitraege" -> "FlashAttention-A2A (Piggybacking)"):
 *   O[b,h,i,:] = softmax_j(scale * q[b,h,i,:] . k[b,h,j,:]) v[b,h,j,:]   (non-causal)
 * followed by the post-attention All-to-All that moves every output row into the sequence
 * shard of its destination rank,
 *   dest[r][b, s_local, h, :] = O[b, h, r*S/P + s_local, :].
 * In the fused call the owner of a finished output tile stores it straight into the
 * destination slabs and goes on with its next tile; no warp or SM is set aside for the
 * exchange.  On one GPU the P ranks are P slabs in local memory.
 *
 * Conventions shared by every call:
 *  - Tensors are bf16 stored as 16-bit words, row-major and contiguous.  q, k, v and the
 *    head-major output use [B, H, S, D]; each destination slab uses [B, S/P, H, D].
 *  - Every pointer named "device" points to memory the caller allocated on the current
 *    CUDA device, 16-byte aligned.  The caller owns all buffers; the library never
 *    allocates, frees or keeps device memory and never synchronises.
 *  - All work is enqueued on `stream` (NULL = legacy default stream) and runs
 *    asynchronously.  Host-detectable errors return before anything is enqueued.
 *  - `dev_status` (nullable) is a device int the kernels set to a non-zero xs_status when a
 *    bounded on-device wait gives up (XS_ERR_TIMEOUT).  The caller zeroes it before the
 *    call and reads it after its own synchronisation.
 *  - Supported shapes: B, H, S, D, P >= 1; H % P == 0 and S % P == 0 (Ulysses sharding);
 *    D % 8 == 0 and 8 <= D <= 128; P <= XS_MAX_RANKS.  S need not be a multiple of the
 *    128-row tile: ragged tails are masked.
 */
#ifndef XS_H_
#define XS_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define XS_API __attribute__((visibility("default")))
#else
#define XS_API
#endif

#define XS_VERSION 100   /* 1.0.0 */
#define XS_MAX_RANKS 16

typedef enum {
  XS_OK = 0,
  XS_ERR_INVALID_ARG = 1, /* null/misaligned/overlapping pointers, non-positive sizes   */
  XS_ERR_UNSUPPORTED = 2, /* shape outside the supported set (see conventions)          */
  XS_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, tensor map, ...) */
  XS_ERR_TIMEOUT = 4      /* written to *dev_status by a bounded on-device wait          */
} xs_status;

/* Problem shape.  B batch, H heads, S sequence length, D head dim, P Ulysses ranks. */
typedef struct {
  int B, H, S, D, P;
} xs_shape;

struct CUstream_st;
typedef struct CUstream_st *xs_stream_t; /* the same handle as cudaStream_t */

/*
 * Fused attention + post-attention All-to-All (the hot path).
 *   q, k, v   : device, [B, H, S, D] bf16.
 *   dest      : HOST array of P device pointers; dest[r] is rank r's slab [B, S/P, H, D].
 *               Slabs must not overlap one another or q, k, v.
 *   scale     : softmax scale; <= 0 selects 1/sqrt(D) with the true D.
 * Numerics: bf16 operands, fp32 accumulation of Q K^T and P V, probabilities rounded to
 * bf16 before P V, fp32 row sums of those rounded probabilities, output rounded to bf16
 * (nearest even).
 * Returns XS_OK once the work is enqueued; errors as listed in xs_status.
 */
XS_API xs_status xs_attn_a2a_fused(const void *q, const void *k, const void *v, void *const *dest,
                            xs_shape shape, float scale, xs_stream_t stream, int *dev_status);

/*
 * The same fused call for one rank of a multi-GPU Ulysses layer (the per-rank piece of the
 * exchange the pages describe: each rank owns a subset of the heads over the full sequence
 * and writes its finished tiles into every rank's sequence shard).
 *   q, k, v     : device, [B, shape.H, S, D]: the shape.H heads this rank owns.
 *   heads_total : heads of the layer; every destination row holds all of them.
 *   head_offset : global index of this rank's first head (rank g of P: g * shape.H).
 *   dest        : HOST array of shape.P slab pointers; dest[r] is [B, S/P, heads_total, D].
 *                 The pointers may be this GPU's memory or memory of other GPUs that this
 *                 GPU can store to (peer access); the call only stores to them.
 * Writes dest[r][b, s_local, head_offset + h, :] = O[b, h, r*S/P + s_local, :] for this
 * rank's heads h; the other heads' columns of the slabs are left untouched.  Requires
 * heads_total % P == 0, S % P == 0 and head_offset + shape.H <= heads_total.
 * xs_attn_a2a_fused(...) equals this call with heads_total = shape.H, head_offset = 0.
 */
XS_API xs_status xs_attn_a2a_fused_rank(const void *q, const void *k, const void *v,
                                        void *const *dest, xs_shape shape, int heads_total,
                                        int head_offset, float scale, xs_stream_t stream,
                                        int *dev_status);

/*
 * xs_attn_a2a_fused_rank that also publishes, per destination slab, an arrival counter: the
 * device-initiated completion signal of the one-sided stores (X-Stage abstract: the exchange
 * is made of device-initiated one-sided remote stores; explainer "FlashAttention-A2A
 * (Piggybacking)": the tile's owner stores it into the destination rank's shard).  Arguments
 * and results as xs_attn_a2a_fused_rank, plus:
 *   slab_flags : HOST array of shape.P device pointers; slab_flags[r] is one 32-bit counter,
 *                4-byte aligned, that lives with slab r (on the GPU that owns it, which may be
 *                another GPU reachable by peer access), outside every slab and input.  Distinct.
 * After storing its rows of a tile, each storing warp adds the number of rows it stored into
 * slab r to *slab_flags[r] with a system-scope release, so a reader that observes the counter
 * with an acquire load also observes those rows.  One complete call adds
 * B * (S / P) * shape.H to every slab's counter.  Counters only grow (mod 2^32): a caller
 * that reuses them across steps waits for the running total (see xs_slab_wait) instead of
 * clearing them, or clears them (cudaMemsetAsync) in stream order before the call.
 * The storing warps wait for their own stores to become visible before each release; this
 * is done by the warps that store, after they have handed the tile's accumulator back, so
 * the attention's key loop does not wait for it.
 */
XS_API xs_status xs_attn_a2a_fused_flags(const void *q, const void *k, const void *v,
                                         void *const *dest, unsigned int *const *slab_flags,
                                         xs_shape shape, int heads_total, int head_offset,
                                         float scale, xs_stream_t stream, int *dev_status);

/*
 * Consumer side of the arrival counters: enqueue on `stream` a wait until *flag has reached
 * `target` (compared modulo 2^32: the wait ends once flag - target, as a signed 32-bit
 * value, is >= 0).  One GPU thread polls the counter with system-scope acquire loads; work
 * enqueued on `stream` after this call sees every row that the counted releases covered.
 *   flag       : device pointer (this GPU's memory or a peer's), 4-byte aligned.
 *   limit_ns   : 1e3 <= limit_ns <= 1e11; after that much global time the wait gives up and
 *                writes XS_ERR_TIMEOUT to *dev_status (device int, required).
 * On one GPU the wait must be ordered after the producing call (same stream, or an event):
 * a waiting kernel and the kernel it waits for are not guaranteed to run at the same time on
 * one device.  Across GPUs the producers run on their own devices.
 */
XS_API xs_status xs_slab_wait(const unsigned int *flag, unsigned int target, long long limit_ns,
                              xs_stream_t stream, int *dev_status);

/*
 * xs_attn_a2a_fused with a record of the sender-visible store-issue span of every output
 * tile (the quantity the X-Stage explainer's Burst-Gap model describes: "Methodik: Die
 * X-Stage-Abstraktion und das Burst-Gap-Modell").  Same arguments and results as
 * xs_attn_a2a_fused, plus:
 *   spans     : device, 8-byte aligned, [n_items][2][4][3] uint64 with n_items = B * H *
 *               ceil(S / 256) work items of 256 query rows (two 128-row tiles), for each
 *               tile and each of the four warps that store it: SM clock (clock64) before the
 *               warp prepares its first store, SM clock after its last store has
 *               been issued (not completed), and the global timer (ns) at the first stamp.
 *   spans_len : words available at spans (>= n_items * 24, else XS_ERR_INVALID_ARG).
 * A separate kernel instance: xs_attn_a2a_fused itself records nothing.
 */
XS_API xs_status xs_attn_a2a_fused_spans(const void *q, const void *k, const void *v,
                                         void *const *dest, xs_shape shape, float scale,
                                         unsigned long long *spans, long long spans_len,
                                         xs_stream_t stream, int *dev_status);

/*
 * Attention only, head-major output: out[b,h,s,:] (device, [B, H, S, D] bf16).  The same
 * kernel and arithmetic as xs_attn_a2a_fused, so out re-laid by xs_a2a_relayout equals the
 * fused result bit for bit.  First half of the serial baseline the pages compare against
 * ("over serial execution", same item of the explainer).  P is only range-checked here.
 */
XS_API xs_status xs_attn(const void *q, const void *k, const void *v, void *out, xs_shape shape,
                  float scale, xs_stream_t stream, int *dev_status);

/*
 * The post-attention All-to-All as a separate pass (second half of the serial baseline):
 *   dest[r][b, s_local, h, :] = src[b, h, r*S/P + s_local, :]
 * src: device [B, H, S, D] 16-bit words; dest: host array of P device slab pointers, each
 * [B, S/P, H, D].  A pure copy: every destination word equals its source word.  Needs
 * S % P == 0 but any H (a GPU holding H/N of a layer's heads packs them per rank with it).
 */
XS_API xs_status xs_a2a_relayout(const void *src, void *const *dest, xs_shape shape,
                          xs_stream_t stream);

/*
 * The pre-attention All-to-All of Ulysses (sequence shards -> head-major; the direction
 * that precedes the attention in the layer the pages fuse the post-attention exchange
 * into):
 *   dst[b, h, r*S/P + s_local, :] = src[r][b, s_local, head_offset + h, :]
 * for h < heads_local (one rank's heads; heads_local = H and head_offset = 0 gathers all).
 * src: host array of P device slab pointers, each [B, S/P, H, D] with H = shape.H (all heads);
 * dst: device [B, heads_local, S, D].  A pure copy of 16-bit words.
 */
XS_API xs_status xs_a2a_pre(void *const *src, void *dst, xs_shape shape, int heads_local,
                            int head_offset, xs_stream_t stream);

/*
 * Partial attention over one key/value shard, with the log-sum-exp of every query row: the
 * owner's side of the Route primitive (page "Move the Query, Not the Cache: Characterizing
 * Cross-Instance Latent Attention Redistribution Across GPU Fabrics", explainer "Technisches
 * Resuemee: Den Query bewegen, nicht den Cache" -> "Methodik" -> "Primitiv-Vergleich": the
 * query is sent to the owner of a KV shard, the owner computes the partial attention there,
 * and the requester merges the small results by online softmax).  Per (b, h) and query row i,
 * over the s_kv keys j of the shard, with s_j = scale * q[b,h,i,:] . k[b,h,j,:]:
 *   o_part[b,h,i,:] = sum_j exp(s_j) v[b,h,j,:] / sum_j exp(s_j)
 *   lse[b,h,i]      = log sum_j exp(s_j)                         (natural log)
 *   q      : device [B, H, S, D] bf16 (S = shape.S query rows);
 *   k, v   : device [B, H, s_kv, D] bf16 (unused, may be NULL, when s_kv == 0);
 *   o_part : device [B, H, S, D] fp32, 16-byte aligned;  lse: device [B, H, S] fp32.
 * shape.P must be 1 (no exchange here); the other shape rules are those of xs_attn, with any
 * s_kv >= 0 (ragged tails masked).  s_kv == 0 (an empty shard) writes o_part = 0 and
 * lse = -inf, which the merge treats as a part of weight zero.  Numerics: as xs_attn (P
 * rounded to bf16 before P V, fp32 accumulation, l summed from the rounded weights), the
 * output kept in fp32 so that the merge adds no bf16 rounding of its own.
 */
XS_API xs_status xs_attn_partial(const void *q, const void *k, const void *v, float *o_part,
                                 float *lse, xs_shape shape, int s_kv, float scale,
                                 xs_stream_t stream, int *dev_status);

/*
 * The requester's merge of n_parts partial results of the same query rows over disjoint key
 * shards (same passage as xs_attn_partial): per row, M = max_t lse_t, w_t = exp(lse_t - M),
 *   out = sum_t w_t o_t / sum_t w_t            (rounded to bf16)
 *   lse_out = M + log(sum_t w_t)               (when lse_out is not NULL)
 * which is the attention over the union of the shards.  Rows whose parts all have
 * lse = -inf give out = 0 and lse_out = -inf; a part with lse = -inf has no weight.
 *   o_parts   : host array of n_parts device pointers, each [rows, D] fp32, 16-byte aligned;
 *   lse_parts : host array of n_parts device pointers, each [rows] fp32;
 *   out       : device [rows, D] bf16;  lse_out: device [rows] fp32 or NULL.
 * 1 <= n_parts <= XS_MAX_PARTS; D % 8 == 0, 8 <= D <= 4096.  Outputs may not overlap inputs.
 * For partial attention results, rows = B * H * S (their [B, H, S] leading dimensions).
 */
#define XS_MAX_PARTS 16
XS_API xs_status xs_lse_merge(const float *const *o_parts, const float *const *lse_parts,
                              int n_parts, void *out, float *lse_out, long long rows, int D,
                              xs_stream_t stream);

/*
 * Burst-Gap store microbenchmark (explainer, "Methodik: Die X-Stage-Abstraktion und das
 * Burst-Gap-Modell": sender-visible issue time T_iss(G; K, V) of a burst of volume V from K
 * producers separated by a compute gap G).  Each of `producers` CTAs repeats n_bursts times:
 * issue its share (burst_bytes / producers) of 16-byte stores into `scratch`, record when
 * the last of its threads has issued, then run a dependent FMA chain of about gap_cycles
 * cycles.  Nothing waits for the stores to complete: the measured time is what the issuer
 * sees.
 *   scratch       : device buffer of scratch_bytes bytes (stored to, never read).
 *                   Bursts walk through it cyclically, so a buffer larger than L2 makes the
 *                   stores drain to HBM.
 *   stamps        : device, [producers, n_bursts, 4] uint64 per burst: SM clock at burst
 *                   start, SM clock when the CTA finished issuing, SM clock at gap end,
 *                   global timer (ns) at burst start.
 * Limits: burst_bytes % (16 * producers) == 0; each producer's share >= 16 bytes and
 * <= scratch_bytes / producers; 1 <= producers <= 4096; 1 <= n_bursts <= 1 << 20;
 * 0 <= gap_cycles <= 1 << 30; threads_per_producer in {32, 64, ..., 1024}.
 */
typedef struct {
  long long burst_bytes;    /* V: aggregate bytes per burst over all producers */
  int producers;            /* K: number of producer CTAs                        */
  long long gap_cycles;     /* G: compute gap after each burst, in SM cycles     */
  int n_bursts;             /* bursts per producer                               */
  int threads_per_producer; /* CTA size                                          */
} xs_burst_cfg;

XS_API xs_status xs_burst_probe(void *scratch, long long scratch_bytes, xs_burst_cfg cfg,
                         unsigned long long *stamps, xs_stream_t stream);

/*
 * Allocation-free variant of xs_burst_probe.  (The pages have no counterpart: this exists for
 * callers of this library, not for the method.)  Some callers cannot call cudaMalloc: a
 * health-check or monitoring hook that runs inside a serving process whose device memory is
 * already reserved by that process's caching allocator (an extra allocation can fail, or
 * force the allocator to release and re-fragment its pool), or a runtime that forbids device
 * allocation once it is initialised.  This entry point lets them run the probe with nothing
 * but the stamps buffer they already own.
 *   - Scratch: a fixed XS_BURST_STATIC_SCRATCH_BYTES (32 MiB) array in the library's own
 *     global memory, held on every GPU that loads the library until the process exits.  The
 *     bursts walk through it cyclically, so they stay L2-resident (32 MiB < L2); for
 *     HBM-drain measurements use xs_burst_probe with a buffer larger than L2.
 *   - burst_bytes above XS_BURST_STATIC_SCRATCH_BYTES is rejected with XS_ERR_UNSUPPORTED;
 *     other limits and the stamps layout are those of xs_burst_probe.
 *   - Every call looks up the array's device address in the CUDA context current on the
 *     calling thread (cudaGetSymbolAddress, which allocates nothing), so callers that switch
 *     contexts or reset the device get the right address.  The first call in a context may
 *     load the library's device code into it: make that first call before any stream
 *     capture.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 *   - Every call shares the one array and leaves its contents behind; the probe only stores
 *     into it, so nothing needs to start at zero.  Calls that overlap on the GPU (other
 *     streams, other threads) race on the array: their stores interleave and each one's
 *     stamps then include the other's traffic.
 */
#define XS_BURST_STATIC_SCRATCH_BYTES (32LL << 20)
XS_API xs_status xs_burst_probe_static(xs_burst_cfg cfg, unsigned long long *stamps,
                                       xs_stream_t stream);

/*
 * Self-test of the bounded on-device wait used by every kernel in this library: launches
 * one thread that waits on a shared-memory barrier nothing ever arrives at, gives up after
 * limit_ns nanoseconds of global time (1e3 <= limit_ns <= 1e10) and writes XS_ERR_TIMEOUT
 * to *dev_status (device, required).  The context stays usable afterwards.
 */
XS_API xs_status xs_selftest_bounded_wait(int *dev_status, long long limit_ns, xs_stream_t stream);

/*
 * Self-test of the attention kernel's own abort path.  Runs xs_attn (head-major output) with
 * two changes: every CTA's TMA producer stops before its fill number `stall_fill` (Q and K/V
 * tile fills of that CTA counted together from 0), as if that copy never arrived, and every
 * on-device wait gives up after limit_ns nanoseconds of global time instead of the
 * library's 2 s.  The waits that depend on the missing fill then run out: the kernel writes
 * XS_ERR_TIMEOUT to *dev_status, each CTA lets the copies and MMAs it already started
 * finish, frees its tensor memory and returns, and the context stays usable.  `out` is left
 * partly written.  Arguments as xs_attn, plus:
 *   stall_fill : >= 0; a CTA that needs fewer fills completes normally.
 *   limit_ns   : 1e3 <= limit_ns <= 1e10.
 *   dev_status : device int, required.
 * A test entry point: no page of the method describes it.
 */
XS_API xs_status xs_selftest_attn_abort(const void *q, const void *k, const void *v, void *out,
                                        xs_shape shape, int stall_fill, long long limit_ns,
                                        xs_stream_t stream, int *dev_status);

/*
 * Peer mapping of destination slabs between the processes of one node (one process per
 * GPU).  In the multi-GPU form of the exchange (X-Stage explainer, "FlashAttention-A2A
 * (Piggybacking)": the tile's owner sends the finished tile to the rank that needs it), each
 * GPU holds the sequence-shard slabs of its own ranks; the other GPUs map them with these
 * calls and pass the mapped pointers in the `dest` array of xs_attn_a2a_fused_rank, whose
 * epilogue then stores straight into them over NVLink.  Nothing is allocated or freed here
 * beyond the mapping itself; no call synchronises a stream.
 */
#define XS_IPC_HANDLE_BYTES 64

/*
 * Export the allocation that contains `ptr` for mapping by other processes.
 *   ptr    : device pointer into memory from cudaMalloc (directly, or through a caching
 *            allocator built on it) on any device of this process.
 *   handle : host buffer of XS_IPC_HANDLE_BYTES bytes; receives the CUDA IPC handle of the
 *            whole allocation (the handle is opaque and valid on this node only).
 *   offset : host; receives ptr minus the allocation's first byte.
 * Errors: XS_ERR_INVALID_ARG for a null argument; XS_ERR_CUDA when the driver refuses (the
 * memory is not a cudaMalloc allocation, e.g. a virtual-memory mapping).  The exporter must
 * keep the memory alive until every process that opened the handle has closed it.
 */
XS_API xs_status xs_ipc_export(const void *ptr, unsigned char *handle, long long *offset);

/*
 * Map an allocation exported by another process of this node.
 *   handle : host, XS_IPC_HANDLE_BYTES bytes from xs_ipc_export in that process.
 *   base   : host; receives the mapped address of the allocation's first byte in this
 *            process (add the exporter's offset to reach its pointer).  Peer access from the
 *            current device to the owning device is enabled on first use.
 * Errors: XS_ERR_INVALID_ARG for a null argument; XS_ERR_CUDA when the driver refuses (the
 * handle came from this same process, or the devices cannot reach each other).
 * Every successful open is paired with one xs_ipc_close(base).
 */
XS_API xs_status xs_ipc_open(const unsigned char *handle, void **base);

/* Unmap a base returned by xs_ipc_open; no kernel that stores through it may still run. */
XS_API xs_status xs_ipc_close(void *base);

/* Human-readable name of a status code (static storage, never NULL). */
XS_API const char *xs_get_error_string(xs_status status);

/* Library version, XS_VERSION of the build. */
XS_API int xs_version(void);

/* Text of the last error the calling thread got from this library (static per thread). */
XS_API const char *xs_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* XS_H_ */
