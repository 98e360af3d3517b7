/*
 * gsparse — residual gradient sparsification for data-parallel SGD on NVIDIA B200 (sm_100a).
 *
 * C ABI of libgsparse.so. Every entry point is a stream-ordered sequence of hand-written CUDA
 * kernels; there is no CPU fallback.
 *
 * Method (web pages on the subject):
 *  - "Sparse Communication for Distributed Gradient Descent" (Aji & Heafield, EMNLP 2017),
 *    Abstract: map the 99% smallest updates by absolute value to zero and exchange the rest as
 *    sparse matrices; the result can be combined with quantisation.
 *  - "Sparse Binary Compression: Towards Distributed Deep Learning with minimal Communication"
 *    (Sattler et al., arXiv 1805.08768v1), §II: communication delay, sparse binarisation,
 *    residual accumulation, Golomb position encoding; Appendix A: decoding needs no shapes.
 *  - "Combining Global Sparse Gradients with Local Gradients in Distributed Neural Network
 *    Training" (Aji, Heafield & Bogoychev, EMNLP-IJCNLP 2019), Abstract: combine the compressed
 *    global gradient with the node's own uncompressed gradient.
 *
 * Conventions shared by all calls
 *  - Pointer arguments are DEVICE pointers owned by the caller, unless a comment says "host".
 *    The library allocates and frees nothing; scratch memory is the caller's `workspace`, whose
 *    required size the matching *_workspace_size() function returns.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream). No call
 *    synchronises the host. Calls that use separate workspaces may run concurrently. The library
 *    keeps no state between calls, with one exception: gsparse_residual_topk_noalloc uses a fixed
 *    scratch array owned by the library, shared by all its calls on a device, so calls of it
 *    that overlap on the GPU must be serialised.
 *  - The return value is a gsparse_status for errors found on the host before any launch (bad
 *    arguments, short workspace, launch failure). Errors that depend on device data are OR-ed as
 *    GSPARSE_DERR_* bits into *d_status (device int32; may be NULL to ignore them). The library
 *    never clears *d_status; kernels that find such an error skip the affected work and never
 *    trap, assert or wait without bound.
 *  - Floating point: fp32 add and multiply are single IEEE round-to-nearest-even operations (no
 *    fused multiply-add); means and sums follow the fixed orders stated below, so results are
 *    bitwise reproducible.
 *  - Index type: int32 flat indices; n must be below 2^31.
 */
#ifndef GSPARSE_H
#define GSPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same types as cudaStream_t and cudaEvent_t. */
typedef struct CUstream_st* gsparse_stream;
typedef struct CUevent_st* gsparse_event;

/* Host-side status. */
enum gsparse_status {
  GSPARSE_OK = 0,
  GSPARSE_ERR_INVALID_ARG = 1, /* null or misaligned pointer, negative size, bad keep fraction */
  GSPARSE_ERR_WORKSPACE = 2,   /* workspace_bytes below the call's minimum */
  GSPARSE_ERR_CUDA = 3,        /* a kernel launch or memset failed (cudaGetLastError) */
  GSPARSE_ERR_UNSUPPORTED = 4  /* n >= 2^31, too many workers, b outside 0..30 */
};

/* Device-side error bits, OR-ed into *d_status. */
enum gsparse_device_error {
  GSPARSE_DERR_CAPACITY = 1,       /* an output array is too small for the result */
  GSPARSE_DERR_CORRUPT_STREAM = 2, /* Golomb stream inconsistent with its length or side table */
  GSPARSE_DERR_INDEX_RANGE = 4,    /* an index outside [0, n) or a list not strictly ascending */
  GSPARSE_DERR_SEGMENTS = 8,       /* segment offsets not ascending from 0 to n */
  GSPARSE_DERR_TIMEOUT = 16        /* a bounded wait for an asynchronous copy gave up (about a
                                      second); the call stopped and its outputs are not valid */
};

/* Flags for gsparse_residual_topk / gsparse_binarize. */
enum gsparse_select_flags {
  GSPARSE_SELECT_DEFAULT = 0,
  /* Skip the sampled candidate threshold: every entry is a candidate and the exact threshold is
     found from the full data. Same result, more memory traffic. */
  GSPARSE_SELECT_EXHAUSTIVE = 1,
  /* gsparse_binarize only: the magnitude-first reading of sparse binarisation (see there). */
  GSPARSE_BINARIZE_BY_MAGNITUDE = 2,
  /* Test hook for the failure path, never for production use: in gsparse_residual_topk and
     gsparse_residual_topk_momentum the first bounded wait of every warp of the streaming pass
     waits on a barrier that nothing completes, with a limit of 2^16 SM cycles. The wait runs
     out, GSPARSE_DERR_TIMEOUT is raised, the rest of the call does nothing, and residual,
     momentum buffer and outputs are left partly updated (not valid); the context stays usable.
     No effect on gsparse_binarize (its streaming pass has no waits). */
  GSPARSE_SELECT_TEST_EXPIRE_WAIT = 4
};

const char* gsparse_status_string(int status);
const char* gsparse_version(void);

/* Per-call measurement events (HOST struct, optional): a call of gsparse_residual_topk,
 * gsparse_residual_topk_momentum or gsparse_binarize given a non-NULL pointer with both events
 * set records `before` on its stream right before its streaming pass over g and the residual,
 * and `after` right after it, so that pass can be timed alone with cudaEventElapsedTime. The
 * events are created by the caller (cudaEventCreate); NULL records nothing. */
typedef struct {
  gsparse_event before;
  gsparse_event after;
} gsparse_pass_events;

/* ---------------------------------------------------------------------------------------------
 * Host helpers.
 */

/* Entries kept from a segment of n_s entries at keep fraction keep_num/keep_den:
 * ceil(n_s * keep_num / keep_den) in exact integer arithmetic, clamped to [0, n_s]. Dropping 99%
 * (Aji & Heafield 2017, Abstract) is keep 1/100. Returns -1 for a bad fraction. */
int64_t gsparse_k_for(int64_t n_s, int64_t keep_num, int64_t keep_den);

/* Golomb parameter for positions of density p: b* = 1 + floor(log2(log(phi-1) / log(1-p))),
 * phi the golden ratio (the rule given with the ResNet-50 sparse-binary workload; Sattler et
 * al., §II Optimal Position Encoding, names Golomb coding of the distances). -1 if p not in (0,1). */
int32_t gsparse_golomb_b_star(double p);

/* Warm-up sparsity schedule ("Sparse Binary Compression", Appendix A: warm-up training raises the
 * sparsity exponentially from 25% to 0.1% kept during the first epochs). READING: the keep
 * fraction at step t of a warm-up of T steps is start * (end / start)^(t / T), and end from step T
 * on. Returned as the numerator of keep = num / den (rounded to nearest, clamped to [1, den]), so
 * the step's selection is gsparse_residual_topk with keep (num, den). -1 for bad arguments
 * (den <= 0, fractions outside (0, 1], negative t or T). */
int64_t gsparse_warmup_keep_num(int64_t t, int64_t T, double start, double end, int64_t den);

/* ---------------------------------------------------------------------------------------------
 * Residual top-k  (Aji & Heafield 2017, Abstract; Sattler et al. §II Residual Accumulation and
 * Communication Delay)
 *
 *   acc_i = fl(g_i + residual_i)
 *   per segment s: send the k_s = gsparse_k_for(n_s, keep) entries of largest |acc_i|, ties to
 *   the lower index (the order of |x| is the order of the fp32 bit pattern with the sign bit
 *   cleared, so +0 and -0 tie and NaN ranks above +inf);
 *   residual_i <- +0.0f for the sent entries, acc_i for all others.
 *
 * g, residual      fp32[n], 16-byte aligned; residual is read and overwritten in place.
 * seg_offsets      int64[num_segments+1] device array of ascending offsets from 0 to n, or NULL
 *                  with num_segments == 1 for one global selection. One segment per tensor gives
 *                  per-tensor selection.
 * keep_num/den     keep fraction, 0 <= keep_num <= keep_den, keep_den > 0. keep_num == 0 only
 *                  accumulates (residual <- fl(g + residual)), the communication-delay step.
 * out_idx, out_val int32/fp32[out_capacity]: sent indices ascending within each segment, segments
 *                  in order, with their acc values.
 * out_offsets      int64[num_segments+1] device: exclusive offsets of each segment's entries.
 * out_capacity     host bound; if sum_s k_s exceeds it, GSPARSE_DERR_CAPACITY is raised and
 *                  neither outputs nor residual are touched.
 * pending          HOST pointer to a list of residual writes applied before the step, or NULL:
 *                  residual[idx_j] <- val_j for every entry j (idx strictly ascending in [0, n)).
 *                  It carries the quantisation error of the previous step (gsparse_quantize's
 *                  feedback_out) into this call, which applies it inside its streaming pass rather
 *                  than as a separate scattered write; the result equals writing it first.
 * workspace        256-byte aligned, at least gsparse_residual_topk_workspace_min(); the
 *                  recommended size is gsparse_residual_topk_workspace_size(). Less room only
 *                  costs speed.
 * pass_events      HOST pointer or NULL: events recorded around the streaming pass (above).
 * Data errors: GSPARSE_DERR_SEGMENTS, GSPARSE_DERR_CAPACITY, GSPARSE_DERR_INDEX_RANGE (a pending
 * list that is not strictly ascending in [0, n)); on any of them nothing is written.
 */
typedef struct {
  const int32_t* idx;      /* device, strictly ascending */
  const float* val;        /* device */
  const int64_t* d_count;  /* device int64: number of entries */
  int64_t capacity;        /* host bound on *d_count */
} gsparse_pending;

size_t gsparse_residual_topk_workspace_size(int64_t n, int32_t num_segments, int64_t keep_num,
                                            int64_t keep_den);
size_t gsparse_residual_topk_workspace_min(int64_t n, int32_t num_segments);
int gsparse_residual_topk(const float* g, float* residual, int64_t n, const int64_t* seg_offsets,
                          int32_t num_segments, int64_t keep_num, int64_t keep_den, int32_t* out_idx,
                          float* out_val, int64_t* out_offsets, int64_t out_capacity,
                          const gsparse_pending* pending, uint32_t flags, void* workspace,
                          size_t workspace_bytes, int32_t* d_status, gsparse_stream stream,
                          const gsparse_pass_events* pass_events);

/* Residual top-k with momentum correction and momentum masking ("Sparse Binary Compression",
 * §II "Momentum Correction, Warm-up Training and Momentum Masking" and Appendix A: the
 * momentum-corrected gradient is added to the residual, and the momentum of the entries that
 * were sent is set to zero):
 *
 *   v_i = fl(fl(momentum * u_i) + g_i);   u_i <- v_i
 *   then gsparse_residual_topk on v in place of g (acc_i = fl(v_i + residual_i));
 *   u_i <- +0.0f for every sent entry.
 *
 * momentum_buf   u, fp32[n], 16-byte aligned, read and overwritten in place; must not alias g or
 *                residual. keep_num == 0 only accumulates (u <- v, residual <- fl(v + residual)).
 * All other arguments, the workspace (same size queries) and the errors are those of
 * gsparse_residual_topk. One streaming pass moves 20 bytes per entry (g, u, r read; u, r written).
 */
int gsparse_residual_topk_momentum(const float* g, float* momentum_buf, float momentum,
                                   float* residual, int64_t n, const int64_t* seg_offsets,
                                   int32_t num_segments, int64_t keep_num, int64_t keep_den,
                                   int32_t* out_idx, float* out_val, int64_t* out_offsets,
                                   int64_t out_capacity, const gsparse_pending* pending,
                                   uint32_t flags, void* workspace, size_t workspace_bytes,
                                   int32_t* d_status, gsparse_stream stream,
                                   const gsparse_pass_events* pass_events);

/* ---------------------------------------------------------------------------------------------
 * Residual top-k without caller-provided scratch  (no counterpart in the pages: this entry point
 * exists for callers, not for the method)
 *
 * Some callers cannot call cudaMalloc or hand over a workspace: code that runs inside a host
 * framework whose caching allocator owns the whole device and budgets every byte (an allocation
 * of our own would fail or fight that allocator), or code invoked from that allocator's own hooks
 * (allocating there would re-enter it). This call needs neither: its scratch is a fixed array of
 * GSPARSE_NOALLOC_SCRATCH_BYTES in the library's own device memory. The array comes into
 * existence when the library's top-k module is first used on a device (with CUDA's lazy module
 * loading, the default, that is the first top-k, binarise or noalloc call on that device, which
 * may be this call itself) and stays until the process exits. A caller whose allocator reserves
 * the whole device should make one call (any size) before the reservation. It allocates nothing.
 *
 * Same result as gsparse_residual_topk with seg_offsets = NULL and num_segments = 1 (one global
 * selection) and flags = 0, bit for bit. The caller still owns g, residual and the outputs.
 * - n above GSPARSE_NOALLOC_MAX_N returns GSPARSE_ERR_UNSUPPORTED before any launch.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture on the device.
 * - All calls on a device share the one array and it keeps the last call's contents; each call
 *   clears the parts that must start at zero. Calls whose kernels overlap on the GPU (concurrent
 *   streams, or several host threads) race on the array: serialise them. The host-side lookup
 *   of the address is itself safe from several threads.
 * - If the lookup fails the call returns GSPARSE_ERR_CUDA and clears the runtime's last error.
 */
#define GSPARSE_NOALLOC_MAX_N (1 << 24)
#define GSPARSE_NOALLOC_SCRATCH_BYTES (16u << 20)
int gsparse_residual_topk_noalloc(const float* g, float* residual, int64_t n, int64_t keep_num,
                                  int64_t keep_den, int32_t* out_idx, float* out_val,
                                  int64_t* out_offsets, int64_t out_capacity, int32_t* d_status,
                                  gsparse_stream stream);

/* ---------------------------------------------------------------------------------------------
 * 2-bit quantisation of a sent list  (Aji & Heafield 2017, Abstract: sparsification combined
 * with quantisation)
 *
 * The list is entries [begin, end) of idx/val, begin = *d_begin (0 if d_begin is NULL) and
 * end = *d_end, both device int64; end - begin <= capacity (host bound).
 *   m+ = mean of the positive values, m- = mean of the negative values (a negative number);
 *   q_j = m+ for val_j > 0, m- for val_j < 0, +0.0f for val_j == +-0 (in neither mean).
 *   Mean = (float)(S / count) with S the fixed-order fp64 sum: list positions (counted from
 *   begin) in blocks of 256, each block summed left to right from +0.0, block sums combined
 *   pairwise level by level (an unpaired last block sum moves up unchanged); no members -> 0.
 * sign_bits   uint32[ceil(capacity/32)]: bit (j % 32) of word j / 32 set iff val_{begin+j} < 0;
 *             words up to ceil((end-begin)/32) are written.
 * d_means     fp32[2] device: {m+, m-}.
 * residual    fp32[n] or NULL: residual[idx_j] <- fl(val_j - q_j), the quantisation error fed back
 *             (Sattler et al. §II Residual Accumulation). Indices outside [0, n) raise
 *             GSPARSE_DERR_INDEX_RANGE and are skipped.
 * feedback_out fp32[capacity] or NULL: feedback_out[j] <- fl(val_j - q_j) (position j counted
 *             from begin), the same error as a contiguous list; handed to the next
 *             gsparse_residual_topk as its pending writes (with idx) it has the effect of the
 *             residual argument without the scattered write.
 * write_dequantized  nonzero: val_j <- q_j in place.
 */
size_t gsparse_quantize_workspace_size(int64_t capacity);
int gsparse_quantize(const int32_t* idx, float* val, const int64_t* d_begin, const int64_t* d_end,
                     int64_t capacity, float* residual, int64_t n, float* feedback_out,
                     uint32_t* sign_bits, float* d_means, int32_t write_dequantized,
                     void* workspace, size_t workspace_bytes, int32_t* d_status,
                     gsparse_stream stream);

/* Segmented 2-bit quantisation: the sub-lists [off[s], off[s+1]) of idx/val for s = 0..T-1
 * (off = d_offsets, device int64[T+1], ascending, 0 <= off[0], off[T] <= capacity; e.g. the
 * out_offsets of a per-tensor gsparse_residual_topk) are quantised as by gsparse_quantize with
 * d_begin = &off[s] and d_end = &off[s+1], each with its own two means, in one call:
 * d_means     fp32[2T] device: {m+_s, m-_s} for each segment s.
 * sign_bits, feedback_out   positions counted from off[0] (bit (j % 32) of word j / 32 is the
 *             sign of entry off[0] + j); residual, write_dequantized as for gsparse_quantize.
 * Offsets that are not ascending within [0, capacity] raise GSPARSE_DERR_CAPACITY and nothing is
 * written. */
size_t gsparse_quantize_segments_workspace_size(int64_t capacity, int32_t num_segments);
int gsparse_quantize_segments(const int32_t* idx, float* val, const int64_t* d_offsets,
                              int32_t num_segments, int64_t capacity, float* residual, int64_t n,
                              float* feedback_out, uint32_t* sign_bits, float* d_means,
                              int32_t write_dequantized, void* workspace, size_t workspace_bytes,
                              int32_t* d_status, gsparse_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Sparse binarisation  (Sattler et al. §II Sparse Binarization)
 *
 *   acc = fl(g + residual); per segment s with k_s = gsparse_k_for(n_s, keep):
 *   P = the k_s largest entries with acc > 0, N = the k_s entries with acc < 0 of largest |acc|
 *   (ties to the lower index; either may hold fewer than k_s entries; zeros are in neither);
 *   mu+ = mean of P, mu- = mean of |N| (fixed-order fp64 sums over each set in ascending index
 *   order, as in gsparse_quantize). The set with the larger mean is sent (ties to P) with the
 *   signed mean m_s = +mu+ or -mu-; nothing is sent if both are empty (m_s = +0).
 *   residual_i <- fl(acc_i - m_s) for the sent entries, acc_i for all others.
 * Arguments as for gsparse_residual_topk, plus:
 * d_mean    fp32[num_segments] device: m_s.
 * out_val   fp32[out_capacity] or NULL: m_s for every sent entry.
 * out_offsets  exclusive offsets of the compacted per-segment outputs (counts vary).
 *
 * flags & GSPARSE_BINARIZE_BY_MAGNITUDE: the magnitude-first reading of the same section (only
 * the largest-magnitude fraction is retained, and the sign with the larger absolute mean decides
 * which values remain): S = the k_s entries of largest |acc| (gsparse_residual_topk's selection);
 * mu+ = mean of the positive members of S, mu- = mean of |acc| over its negative members (the
 * fixed-order sums over the positions of S, as gsparse_quantize's means); the members of the
 * larger-mean sign are sent with the signed mean (ties to positive); residual_i <- fl(acc_i - m_s)
 * on them and acc_i everywhere else, the unsent members of S included. Same workspace queries.
 */
size_t gsparse_binarize_workspace_size(int64_t n, int32_t num_segments, int64_t keep_num,
                                       int64_t keep_den);
size_t gsparse_binarize_workspace_min(int64_t n, int32_t num_segments, int64_t keep_num,
                                      int64_t keep_den);
int gsparse_binarize(const float* g, float* residual, int64_t n, const int64_t* seg_offsets,
                     int32_t num_segments, int64_t keep_num, int64_t keep_den, int32_t* out_idx,
                     float* out_val, float* d_mean, int64_t* out_offsets, int64_t out_capacity,
                     uint32_t flags, void* workspace, size_t workspace_bytes, int32_t* d_status,
                     gsparse_stream stream, const gsparse_pass_events* pass_events);

/* ---------------------------------------------------------------------------------------------
 * Golomb position coding  (Sattler et al. §II Optimal Position Encoding; Appendix A)
 *
 * Encodes the ascending indices idx[begin..end) (begin/end as in gsparse_quantize):
 *   gaps d_0 = i_0 - base, d_j = i_j - i_{j-1} - 1 (must be >= 0, else GSPARSE_DERR_INDEX_RANGE);
 *   with M = 2^b: q = d >> b one-bits, one zero-bit, then d mod M in b bits, most significant
 *   first. Stream bit t is bit (t % 32) of words[t / 32]; bits past the end are zero.
 * words       uint32[word_capacity]; a longer stream raises GSPARSE_DERR_CAPACITY.
 * d_nbits     uint64 device: stream length in bits.
 * chunk_table int64[2 * ceil(capacity / chunk)] or NULL: for codeword c*chunk, {bit offset,
 *             preceding index} (base - 1 before codeword 0). Side information for parallel
 *             decoding; not part of the stream.
 * b           0..30.
 */
/* Recommended side-table chunk for a list of up to `capacity` codewords: the largest power of
 * two in [4, 64] that still gives at least 16384 chunks (one decoding thread each), so short
 * lists are decoded by enough threads and long ones keep a small table (16 bytes per chunk).
 * Returns 4 for capacity <= 0. Any chunk >= 1 is valid; this only chooses speed. */
int32_t gsparse_golomb_chunk_hint(int64_t capacity);

size_t gsparse_golomb_encode_workspace_size(int64_t capacity);
int gsparse_golomb_encode(const int32_t* idx, const int64_t* d_begin, const int64_t* d_end,
                          int64_t capacity, int64_t base, int32_t b, uint32_t* words,
                          int64_t word_capacity, uint64_t* d_nbits, int64_t* chunk_table,
                          int32_t chunk, void* workspace, size_t workspace_bytes,
                          int32_t* d_status, gsparse_stream stream);

/* Decodes *d_count codewords (<= capacity) from the first *d_nbits bits of words (uint32[word_
 * capacity]; a length beyond 32 * word_capacity bits is a corrupt stream) into out_idx.
 * With chunk_table (as written by the encoder with the same chunk) the chunks decode in
 * parallel; with NULL one thread decodes sequentially. A codeword running past *d_nbits, bits
 * left over, or a chunk that does not end where the side table says raise
 * GSPARSE_DERR_CORRUPT_STREAM; an index >= n_limit raises GSPARSE_DERR_INDEX_RANGE. */
int gsparse_golomb_decode(const uint32_t* words, int64_t word_capacity, const uint64_t* d_nbits,
                          const int64_t* d_count, int64_t capacity, int64_t base, int32_t b,
                          const int64_t* chunk_table, int32_t chunk, int64_t n_limit,
                          int32_t* out_idx, int32_t* d_status, gsparse_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Scatter-accumulate of W workers' sparse updates  (Aji, Heafield & Bogoychev 2019, Abstract:
 * the compressed global gradient; Sattler et al. §I: the updates of all clients are summed)
 *
 *   G_i = (((+0 + v_{0,i}) + v_{1,i}) + ...) over the workers holding i, in worker order, one fp32
 *   add each. merged output = the ascending union of the indices with their G_i.
 */
typedef struct {
  const int32_t* idx;         /* device, strictly ascending */
  const float* val;           /* device values, or NULL: every entry takes *uniform_val */
  const float* uniform_val;   /* device scalar, read when val is NULL (binarised updates) */
  const int64_t* d_count;     /* device int64: number of entries */
  int64_t capacity;           /* host bound on *d_count */
} gsparse_list;

#define GSPARSE_MAX_WORKERS 64

/* lists: HOST array of W descriptors (1 <= W <= GSPARSE_MAX_WORKERS).
 * dense_out   fp32[n] or NULL: G (untouched entries +0).
 * merged_idx, merged_val, d_merged_count   int32/fp32[merged_capacity] + device int64, or all
 *             NULL. More than merged_capacity entries raise GSPARSE_DERR_CAPACITY.
 * Indices outside [0, n) or lists not strictly ascending raise GSPARSE_DERR_INDEX_RANGE. */
size_t gsparse_scatter_accumulate_workspace_size(int32_t W, int64_t n);
int gsparse_scatter_accumulate(const gsparse_list* lists, int32_t W, int64_t n, float* dense_out,
                               int32_t* merged_idx, float* merged_val, int64_t* d_merged_count,
                               int64_t merged_capacity, void* workspace, size_t workspace_bytes,
                               int32_t* d_status, gsparse_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Receive side in one pass: scatter-accumulate fused with the combination  (Aji, Heafield &
 * Bogoychev 2019, Abstract)
 *
 * out = the result of gsparse_combine_local(G, L, out, n, alpha, beta, mode, own list) with G the
 * result of gsparse_scatter_accumulate(lists, W, n), bit for bit, without writing G to memory:
 * per tile of 8192 indices the worker-ordered sum is formed in shared memory and the combined
 * gradient streamed out, so the call moves 8n bytes plus the lists instead of 20n.
 * mode 0: out_i = fl(fl(alpha * G_i) + fl(beta * L_i)); mode 1: G_i becomes fl(G_i - s_i) on the
 * entries of lists[own] (the worker's own sent update) first.
 * L, out fp32[n], 16-byte aligned, not aliased with each other. dense_out fp32[n] or NULL: also
 * receives G. Device errors as for gsparse_scatter_accumulate.
 */
size_t gsparse_accumulate_combine_workspace_size(int32_t W, int64_t n);
int gsparse_accumulate_combine(const gsparse_list* lists, int32_t W, int64_t n, const float* L,
                               float* out, float alpha, float beta, int32_t mode, int32_t own,
                               float* dense_out, void* workspace, size_t workspace_bytes,
                               int32_t* d_status, gsparse_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Combination with the local gradient  (Aji, Heafield & Bogoychev 2019, Abstract)
 *
 * mode 0 (sum):     out_i = fl(fl(alpha * G_i) + fl(beta * L_i))
 * mode 1 (partial): the same, with G_i replaced by fl(G_i - s_i) on the worker's own sent
 *                   entries (own_idx/own_val, *d_own_count <= own_capacity), so its own
 *                   contribution enters only through L.
 * G, L, out fp32[n], 16-byte aligned (out may alias G or L in mode 0).
 */
int gsparse_combine_local(const float* G, const float* L, float* out, int64_t n, float alpha,
                          float beta, int32_t mode, const int32_t* own_idx, const float* own_val,
                          const int64_t* d_own_count, int64_t own_capacity, int32_t* d_status,
                          gsparse_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* GSPARSE_H */
