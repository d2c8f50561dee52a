/*
 * attn.h - C ABI of libattn: exact blockwise self-attention forward on NVIDIA B200
 * (sm_100a), and the merge of partial results.
 *
 * What is computed. For every batch b, query head h and query row i:
 *     s_j   = scale * <q[b,h,i,:], k[b,g,j,:]>   over the visible keys j,
 *     O_i   = sum_j softmax(s)_j * v[b,g,j,:],
 *     LSE_i = ln(sum_j exp(s_j)),
 * with g = h / (Hq / Hkv). This is the conventional three-step attention
 * ("FlashAttention by hand": logits, a softmax row that sums to one, weights times
 * values), reached exactly, up to floating-point rounding, by the tiled online
 * softmax the same page describes: key/value tiles streamed through on-chip
 * memory, a running maximum and denominator, rescaling of the partial output when
 * the maximum grows, and one final division. The score matrix never reaches
 * global memory.
 *
 * Masking. With causal != 0, key j is visible to query i when
 * kv_off + j <= q_off + i (global positions; HOF SWIFT Attention, section 3,
 * Transform stage names causal masking). A row with no visible key has O = 0 and
 * LSE = -inf.
 *
 * Layouts. q, k, v are bf16, row-major [B][H][N][d] (d contiguous). O is fp32
 * [B][Hq][Nq][d]; LSE is fp32 [B][Hq][Nq], natural log, scale included.
 *
 * Ownership and execution. The caller owns every buffer; the library allocates no
 * device memory. All pointers named "device" must be device (or managed) memory.
 * Calls enqueue work on `stream` (a cudaStream_t; NULL is the legacy default
 * stream) and return without waiting. Buffers must stay valid until that work has
 * finished. No call throws; every call returns an attn_status_t.
 *
 * Errors. Arguments are checked before anything is launched: null or misaligned
 * pointers, non-positive sizes, Hq not a multiple of Hkv, outputs overlapping
 * inputs, a negative or non-finite scale, and offsets/leading dimensions that do
 * not fit give ATTN_ERR_INVALID_ARG. Shapes the kernels are not built for (d other
 * than 64 or 128, more than ATTN_MAX_MERGE_PARTS parts, sizes beyond the tensor-map
 * limits) give ATTN_ERR_UNSUPPORTED. A failed CUDA call gives ATTN_ERR_CUDA. NaN or
 * Inf inside the rows a call attends is not checked and gives unspecified results.
 *
 * Device-side failures. Every wait inside the kernels is bounded (4 s of wall-clock
 * time). A wait that runs out stops the kernel early, leaves its outputs unspecified
 * and is recorded in a per-device status word; the launch itself has already returned
 * ATTN_OK by then. Results therefore count only once attn_device_status has reported
 * ATTN_OK for the stream they were computed on. Nothing traps or faults.
 */
#ifndef ATTN_H
#define ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,
  ATTN_ERR_UNSUPPORTED = 2,
  ATTN_ERR_CUDA = 3,
  ATTN_ERR_TIMEOUT = 4,
  ATTN_ERR_INJECTED = 5
} attn_status_t;

#define ATTN_MAX_MERGE_PARTS 64
#define ATTN_MAX_BATCH_PAIRS 48

/* One (query chunk, key/value chunk) pair of attn_fwd_partial_batch. Rows count in the
 * parent tensors; o and lse are the pair's own outputs (or accumulators). */
typedef struct {
  int64_t q_start, q_len;   /* query rows [q_start, q_start + q_len) */
  int64_t kv_start, kv_len; /* key/value rows [kv_start, kv_start + kv_len) */
  int64_t q_off, kv_off;    /* global positions of the first rows (causal test) */
  float* o;                 /* device, fp32 [B][Hq][q_len][d], 16-byte aligned */
  float* lse;               /* device, fp32 [B][Hq][q_len], 4-byte aligned */
} attn_pair_t;

/* Static description of a status code. Never NULL. */
const char* attn_status_string(int status);

/* ABI version: (major << 16) | minor. */
int attn_version(void);

/*
 * attn_fwd - single-pass attention over a whole sequence ("FlashAttention by hand",
 * paragraphs on the fused tiled computation, the running statistics, rescaling and
 * the final division).
 *
 *   q      device, bf16 [B][Hq][N][d], 16-byte aligned
 *   k, v   device, bf16 [B][Hkv][N][d], 16-byte aligned
 *   o      device, fp32 [B][Hq][N][d], 16-byte aligned (written)
 *   lse    device, fp32 [B][Hq][N], 4-byte aligned (written)
 *   B, Hq, Hkv >= 1 with Hq % Hkv == 0; N >= 1; d in {64, 128}
 *   causal 0 or 1 (key j visible to query i iff j <= i)
 *   scale  finite, >= 0 (normally 1/sqrt(d))
 *   stream cudaStream_t to enqueue on
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, float* o, float* lse,
                       int B, int Hq, int Hkv, int64_t N, int d, int causal, float scale,
                       void* stream);

/*
 * attn_fwd_partial - attention of one query chunk against one key/value chunk: one
 * ring step of Ring Attention ("Ring Attention with Blockwise Parallel
 * Transformers", section 3: each device attends its query block to the key/value
 * block it currently holds), or one fragment of the ATTENTION2D query x key/value
 * grid (section 3: fragment-local statistics). The result is the NORMALISED
 * partial output over this chunk's visible keys plus its LSE, ready for
 * attn_merge.
 *
 *   q        device, bf16: &Q[0][0][q_start][0] of a parent tensor
 *            [B][Hq][q_ld][d]; the chunk is rows [q_start, q_start + Nq)
 *   k_chunk, v_chunk
 *            device, bf16: &K[0][0][kv_start][0] of parents [B][Hkv][kv_ld][d];
 *            the chunk is rows [kv_start, kv_start + Nkv); rows beyond it are
 *            never read
 *   o_part   device, fp32 dense [B][Hq][Nq][d] (written)
 *   lse_part device, fp32 dense [B][Hq][Nq] (written)
 *   q_ld >= Nq, kv_ld >= Nkv: allocated sequence length of the parents
 *   q_off, kv_off >= 0: global position of the chunks' first rows (used only for
 *            the causal test kv_off + j <= q_off + i)
 *   other arguments as for attn_fwd. All pointers 16-byte aligned (lse_part 4).
 */
attn_status_t attn_fwd_partial(const void* q, const void* k_chunk, const void* v_chunk,
                               float* o_part, float* lse_part, int B, int Hq, int Hkv,
                               int64_t Nq, int64_t Nkv, int64_t q_ld, int64_t kv_ld,
                               int64_t q_off, int64_t kv_off, int d, int causal,
                               float scale, void* stream);

/*
 * attn_fwd_partial_acc - attn_fwd_partial fused with the merge: o_acc and lse_acc
 * hold, on entry, a normalised partial result over keys disjoint from this chunk
 * (LSE = -inf with O = 0 where no key has been seen yet), and on exit the
 * combination of that partial with this chunk's, by the same log-sum-exp rule as
 * attn_merge. This is the running update a Ring Attention device applies at each
 * ring step ("Ring Attention with Blockwise Parallel Transformers", section 3) and the
 * rescale of the online softmax ("FlashAttention by hand", paragraphs on the running
 * statistics and rescaling) applied at chunk granularity; it needs no buffer for the
 * chunk's own partial and no separate merge launch. A chunk none of whose keys is
 * visible to a row leaves that row unchanged.
 *
 *   o_acc, lse_acc  device, fp32 [B][Hq][Nq][d] and [B][Hq][Nq], read and written
 *   other arguments exactly as for attn_fwd_partial.
 * Successive calls on one accumulator must be ordered (one stream); calls on
 * different accumulators may run concurrently.
 */
attn_status_t attn_fwd_partial_acc(const void* q, const void* k_chunk, const void* v_chunk,
                                   float* o_acc, float* lse_acc, int B, int Hq, int Hkv,
                                   int64_t Nq, int64_t Nkv, int64_t q_ld, int64_t kv_ld,
                                   int64_t q_off, int64_t kv_off, int d, int causal,
                                   float scale, void* stream);

/*
 * attn_fwd_partial_batch - several pairs of attn_fwd_partial (accumulate = 0) or of
 * attn_fwd_partial_acc (accumulate = 1) over the same parent tensors in ONE launch:
 * e.g. all the chunk pairs of a ring step, or of a whole emulated ring. Each pair's
 * result is exactly that of the single-pair call; the work units of all pairs share
 * one persistent grid, heaviest first, so the tail of one pair is filled by the next.
 *
 *   q      device, bf16 parent [B][Hq][q_ld][d];  k, v: parents [B][Hkv][kv_ld][d]
 *   pairs  HOST array of n_pairs (1 .. ATTN_MAX_BATCH_PAIRS) pair descriptions; every
 *          chunk must lie inside its parent; no two pairs' outputs may overlap
 *   other arguments as for attn_fwd_partial. Rows of a parent outside a pair's chunks
 *   may hold anything, NaN and Inf included (uninitialised memory, or a copy still in
 *   flight): a pair reads them into its last tiles but they never reach its result
 *   (keys there are masked, their value rows are zeroed on chip before P.V, and query
 *   rows there are not stored).
 */
attn_status_t attn_fwd_partial_batch(const void* q, const void* k, const void* v, int B,
                                     int Hq, int Hkv, int64_t q_ld, int64_t kv_ld, int d,
                                     int causal, float scale, const attn_pair_t* pairs,
                                     int n_pairs, int accumulate, void* stream);

/*
 * attn_merge - combine partial results computed over disjoint key sets
 * (ATTENTION2D, section 3: fragment-local statistics normalised and summed in
 * stages; section 2: the combination is commutative and associative, so no
 * approximation enters). Per row, with M = max_i LSE_i and w_i = exp(LSE_i - M):
 *     O = sum_i w_i O_i / sum_i w_i,   LSE = M + ln(sum_i w_i).
 * Parts with LSE = -inf contribute nothing; if all are -inf, O = 0, LSE = -inf.
 * n_parts = 1 copies. The result does not depend on the order of the parts beyond
 * fp32 rounding.
 *
 *   o_parts, lse_parts  HOST arrays of n_parts DEVICE pointers: fp32 [rows][d]
 *                       (32-byte aligned: rows move as 256-bit loads) and fp32
 *                       [rows] (4-byte aligned)
 *   n_parts             1 .. ATTN_MAX_MERGE_PARTS
 *   o, lse              device, fp32 [rows][d] (32-byte aligned) and [rows]
 *                       (written); must not overlap any part
 *   rows >= 1; d in {64, 128}
 */
attn_status_t attn_merge(const float* const* o_parts, const float* const* lse_parts,
                         int n_parts, float* o, float* lse, int64_t rows, int d,
                         void* stream);

/*
 * attn_ring_fwd_host - Ring Attention's schedule on one GPU, from HOST buffers to
 * HOST buffers ("Ring Attention with Blockwise Parallel Transformers", section 3:
 * the sequence is cut into blocks; at ring step s the holder of query block i
 * attends key/value block (i - s) mod n_chunks, and its partial results are
 * combined). The sequence is cut into n_chunks chunks of C = N / n_chunks rows;
 * query chunk i attends, in ring order, every key/value chunk (under the causal
 * mask only chunks 0..i); each pair is one partial (attn_fwd_partial_batch
 * launches) and a query chunk's partials are combined in ring order with
 * attn_merge. Results equal those of the same calls made on device buffers.
 *
 * The copies are pipelined with the compute: the chunks of q, k, v go to the device
 * on h2d_stream as strided copies (causal: Q_0, K_0 V_0, Q_1, K_1 V_1, ...; else all
 * of K, V first, then Q_0, Q_1, ...), every pair is launched as soon as both of its
 * chunks are in, and a query chunk's merged result goes back on d2h_stream as soon
 * as it is final. The call is asynchronous like the others; the work is ordered
 * after earlier work on `stream`, and later work on `stream` waits for all of it,
 * including the last copy back.
 *
 *   q_h, k_h, v_h   HOST, bf16 [B][Hq][N][d], [B][Hkv][N][d]; page-locked memory
 *                   lets the copies overlap (pageable memory works, unoverlapped)
 *   o_h, lse_h      HOST, fp32 chunk-major [n_chunks][B][Hq][C][d] and
 *                   [n_chunks][B][Hq][C] (written)
 *   q_d, k_d, v_d   DEVICE staging, same shapes as q_h, k_h, v_h (16-byte aligned);
 *                   their contents on entry do not matter (a pair may run before the
 *                   neighbouring chunk has arrived; see attn_fwd_partial_batch)
 *   o_d, lse_d      DEVICE, same shapes as o_h, lse_h (o_d 32-byte aligned)
 *   ws_o, ws_lse    DEVICE partial buffers, ws_slots slots of [B][Hq][C][d] and
 *                   [B][Hq][C] (ws_o 32-byte aligned); ws_slots must be at least
 *                   the number of chunks a query chunk visits when that is more than
 *                   one (n_chunks), else 0 and the pointers may be NULL
 *   n_chunks        1 .. ATTN_MAX_BATCH_PAIRS, dividing N
 *   h2d_stream, d2h_stream  streams for the two copy directions (NULL: `stream`)
 *   other arguments as for attn_fwd. Device buffers must not overlap each other.
 * The host buffers are read and written by copies that run after the call returns:
 * they must stay allocated (and q_h, k_h, v_h unchanged) until `stream` has passed
 * this call's work.
 */
attn_status_t attn_ring_fwd_host(const void* q_h, const void* k_h, const void* v_h,
                                 float* o_h, float* lse_h, void* q_d, void* k_d, void* v_d,
                                 float* o_d, float* lse_d, float* ws_o, float* ws_lse,
                                 int ws_slots, int B, int Hq, int Hkv, int64_t N, int d,
                                 int n_chunks, int causal, float scale, void* stream,
                                 void* h2d_stream, void* d2h_stream);

/*
 * attn_ring_fwd_host_noalloc - attn_ring_fwd_host for callers that cannot allocate
 * device memory. The pages have no counterpart of this call: it exists for programs in
 * which cudaMalloc is not an option, for example code in a process whose device memory
 * belongs to another allocator (a framework's caching allocator, a fixed per-component
 * budget), or code on a latency-critical path where an allocation would synchronise the
 * device. It takes the same host inputs and outputs as attn_ring_fwd_host and runs the
 * same kernels in the same order (results are identical), but its device staging
 * buffers and partial slots live in one fixed array of the library's own device data:
 * it calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * The array holds ATTN_NOALLOC_SCRATCH_BYTES bytes, and every GPU on which the library
 * is loaded keeps it until the process exits. A call needs, each piece rounded up to
 * 256 bytes, with C = N / n_chunks and S = n_chunks if n_chunks > 1, else 0:
 *     B*Hq*N*d*2 + 2 * B*Hkv*N*d*2 + B*Hq*N*d*4 + B*Hq*N*4 + S*B*Hq*C*d*4 + S*B*Hq*C*4
 * bytes; a call that needs more returns ATTN_ERR_UNSUPPORTED before touching the
 * device. Invalid arguments give ATTN_ERR_INVALID_ARG as for attn_ring_fwd_host.
 *
 * The first call on a device, with that device current, looks up the array's device
 * address (once per device); make that first call before any stream capture. Every
 * call shares the array, which keeps what the last call left in it; no part of it
 * needs to start at zero, since a call writes every byte it uses before reading it.
 * Calls whose work overlaps on the GPU race on the array: issue them on one stream
 * (later calls on a stream wait for all the work of earlier ones, copies back
 * included) or otherwise order them.
 *
 *   q_h, k_h, v_h, o_h, lse_h, B, Hq, Hkv, N, d, n_chunks, causal, scale, stream,
 *   h2d_stream, d2h_stream: as for attn_ring_fwd_host
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (64ull * 1024ull * 1024ull)
attn_status_t attn_ring_fwd_host_noalloc(const void* q_h, const void* k_h, const void* v_h,
                                         float* o_h, float* lse_h, int B, int Hq, int Hkv,
                                         int64_t N, int d, int n_chunks, int causal,
                                         float scale, void* stream, void* h2d_stream,
                                         void* d2h_stream);

/*
 * attn_device_status - synchronise `stream` and report whether any kernel of this
 * library on the current device recorded a device-side failure since the last
 * reset (ATTN_ERR_TIMEOUT: a bounded wait ran out; the kernel then stopped its
 * work and returned, leaving its outputs unspecified). reset != 0 clears the
 * record. Returns ATTN_ERR_CUDA if synchronising fails.
 */
attn_status_t attn_device_status(void* stream, int reset);

/*
 * attn_debug_inject - host-side fault injection for tests of error paths: the next
 * `count` calls of an entry point that launches work return `status`
 * (which must be a failure code) after argument checks and before any launch.
 * count = 0 disarms. Not thread-safe; for tests only.
 */
attn_status_t attn_debug_inject(int status, int count);

/*
 * attn_debug_wait_timeout - failure-path check for tests: launches one tiny kernel
 * whose single waiting thread waits, through the same bounded mbarrier wait the
 * attention kernel uses, on a barrier that nothing arrives on, with a limit of
 * limit_cycles SM clock cycles at the device's peak clock (1 .. 2^31; converted to
 * wall-clock time, as the kernels' own limit is). The wait runs out, the kernel
 * records ATTN_ERR_TIMEOUT in the device status word (see attn_device_status) and
 * returns; the device stays usable. Nothing traps or faults.
 */
attn_status_t attn_debug_wait_timeout(int64_t limit_cycles, void* stream);

/*
 * attn_debug_exp2 - check of the two exponentials the softmax uses, for tests:
 * y[i] = 2^x[i] through the FMA-pipe polynomial (use_poly = 1: Cody and Waite's
 * reduction to x = n + f, |f| <= 1/2, and a degree-3 minimax polynomial for 2^f, max
 * relative error 7.5e-5 for -125.5 <= x <= 127; just above -126 the result can come
 * out denormal, off by at most 2^-138 in absolute terms) or through the exp unit's
 * ex2.approx (use_poly = 0). The polynomial clamps x below at -126 (it gives at most
 * 2^-125 there, not 0). x, y: device fp32 arrays of n >= 1 values, not overlapping.
 */
attn_status_t attn_debug_exp2(const float* x, float* y, int64_t n, int use_poly, void* stream);

/* Number of CUDA kernels this library has launched in this process (all devices). */
uint64_t attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
