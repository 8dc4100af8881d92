/*
 * ag.h -- C ABI of libag, pair-bias multi-query attention for B200 (sm_100a).
 *
 * The operation is the sequence attention of the page "Making Full-Context
 * AlphaGenome Fit on an RTX 3090" (section "Why stock FlashAttention was not
 * a drop-in replacement", Eq. L_ij): eight query heads share one K/V head,
 * a compact learned pair bias with one cell per 16 x 16 position square is
 * added to the scaled dot product, the sum is soft-capped with cap*tanh(./cap)
 * and a softmax over all keys weights V.  The per-head compact bias comes
 * from a linear projection of a compact pair representation (same page,
 * section "Profiling pointed at one very large object").
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise,
 *     row-major, densely packed.  The caller allocates and owns all inputs
 *     and outputs.  The library allocates no device memory: calls keep no
 *     state on the device besides the error word below (and the static array
 *     of ag_attn_fwd_noalloc), so independent calls may run concurrently on
 *     different streams.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream: AG_OK means the work
 *     was enqueued.  Faults inside a kernel surface at the caller's next
 *     synchronisation, and bounded-wait timeouts in the device error word
 *     (ag_device_error).
 *   - Arguments are validated before anything is launched.  On any error
 *     the call returns the status and writes nothing.
 *   - Outputs must not overlap inputs (AG_ERR_ALIAS).
 *   - The kernels are built for sm_100a only; on any other device the
 *     compute entry points return AG_ERR_UNSUPPORTED.
 */
#ifndef AG_H_
#define AG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AG_OK = 0,
    AG_ERR_NULL = 1,        /* a required pointer is NULL                     */
    AG_ERR_SHAPE = 2,       /* a size is negative or sizes are inconsistent   */
    AG_ERR_ALIGN = 3,       /* a pointer lacks the alignment stated below     */
    AG_ERR_UNSUPPORTED = 4, /* valid sizes the kernels do not handle, or the
                               current device is not sm_100                   */
    AG_ERR_VALUE = 5,       /* a scalar argument is out of range (cap)        */
    AG_ERR_CUDA = 6,        /* a CUDA runtime or driver call failed           */
    AG_ERR_ALIAS = 7,       /* an output buffer overlaps an input buffer      */
    AG_ERR_DEVICE = 8,      /* the device error word is set (see below)       */
    AG_ERR_SCRATCH = 9      /* ag_attn_fwd_noalloc: the call needs more scratch
                               than its static buffer holds                   */
} ag_status;

/* Static, human-readable name of a status code (never NULL). */
const char *ag_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int ag_version(void);

/*
 * ag_pair_bias_project -- compact pair representation to per-head bias.
 *
 *   bias[h, p, q] = sum_c pair[p, q, c] * W[c, h]
 *
 * Source: page "Making Full-Context AlphaGenome Fit on an RTX 3090", section
 * "Profiling pointed at one very large object" (the dense path projects a
 * compact pair representation into the attention bias before repeating it
 * 16x along both sequence axes).  The page gives no further terms; this is
 * the plain linear map.
 *
 *   pair  [P, P, Cp] float32, 16-byte aligned
 *   W     [Cp, H]    float32,  4-byte aligned
 *   bias  [H, P, P]  float32,  8-byte aligned (written)
 *   P >= 0 (P == 0 is a no-op); supported: Cp == 128, H == 8, P <= 4096.
 * Float32 multiply-add accumulation in a fixed order.
 */
ag_status ag_pair_bias_project(const float *pair, const float *W, float *bias,
                               int64_t P, int64_t Cp, int64_t H, void *stream);

/*
 * ag_pair_bias_project_rows -- the same projection for R rows of the pair
 * representation (R <= P), e.g. the rows of the query positions one GPU
 * holds when the queries are split between GPUs (see
 * ag_attn_fwd_query_slab):
 *   pair [R, P, Cp] -> bias [H, R, P],  bias[h, r, q] = sum_c pair[r, q, c] W[c, h]
 * Same types, alignment and statuses as ag_pair_bias_project (R > 4096 is
 * AG_ERR_UNSUPPORTED, R < 0 AG_ERR_SHAPE, R == 0 a no-op);
 * ag_pair_bias_project is this call with R = P.
 */
ag_status ag_pair_bias_project_rows(const float *pair, const float *W, float *bias,
                                    int64_t R, int64_t P, int64_t Cp, int64_t H,
                                    void *stream);

/*
 * ag_attn_fwd -- fused pair-bias multi-query attention forward.
 *
 * For b < B, h < H, query i < L, key j < L (page "Making Full-Context
 * AlphaGenome Fit on an RTX 3090", section "Why stock FlashAttention was not
 * a drop-in replacement", Eq. L_ij; online softmax of section "Online
 * softmax, one block at a time"):
 *   s_ij   = q[b,h,i,:] . k[b,j,:] / sqrt(D) + bias[h, i/block, j/block]
 *   L_ij   = cap * tanh(s_ij / cap)       (cap == +INFINITY: L_ij = s_ij)
 *   lse    = log(sum_j exp(L_ij))         (natural log)   -> lse[b,h,i]
 *   out    = sum_j exp(L_ij - lse) v[b,j,:]              -> out[b,h,i,:]
 * No L x L tensor is formed.  No mask (every key attends).
 *
 *   q     [B, H, L, D]  bfloat16 bit patterns, 16-byte aligned
 *   k     [B, L, D]     bfloat16, 16-byte aligned (one head, shared by all H)
 *   v     [B, L, D]     bfloat16, 16-byte aligned (one head, shared by all H)
 *   bias  [H, P, P]     float32,   4-byte aligned, P = ceil(L / block),
 *                       shared by every batch item (one bias per item:
 *                       ag_attn_fwd_strided_bias)
 *   out   [B, H, L, D]  float32,  16-byte aligned (written)
 *   lse   [B, H, L]     float32,   4-byte aligned (written)
 *   cap   > 0 and not NaN; +INFINITY disables the soft cap.
 * Supported: H == 8, D == 128, block == 16, any L <= 65536 (a length that
 * is not a multiple of 16 ends in a partial block, which uses its compact
 * bias cell like the others: the page lists tails among what its kernel does
 * not support yet, section "What has not yet been demonstrated"),
 * B * L <= 2^28 and B * ceil(ceil(L/16)/2) * ceil(L/128) <= 2^30 (B * L^2 up
 * to about 2^42).  B == 0 or L == 0 is a no-op (pointers may be NULL).
 * Products in bf16 with fp32 accumulation (tensor cores); softmax in fp32;
 * the probabilities are rounded to bf16 for the second product while the
 * row sums use their fp32 values.
 *
 * Schedule: the kernel runs one 2-CTA cluster per SM pair, each taking
 * whole pairs of 16-position query blocks.  When those do not divide evenly
 * over the SM pairs (e.g. L = 8192, B = 1: 256 pairs on 74 SM pairs), some
 * pairs have their keys split in two: the first piece runs in the first
 * launch and writes its normalised partial result to out/lse, the second
 * piece runs in a second launch on the same stream (programmatic dependent
 * launch, so it starts on the SMs the first launch frees) and merges the
 * first piece's result with its own by log-sum-exp.  No scratch memory is
 * used, so calls on different streams may overlap freely.  The softmax
 * shifts by a fixed amount for cap <= 60 (the soft cap bounds every logit);
 * for a larger cap or no cap (value width 128) a first pass writes every
 * row's largest logit into lse and the main kernel then shifts each row by
 * it, over whole pairs (value width 192: a running maximum).
 */
ag_status ag_attn_fwd(const void *q, const void *k, const void *v,
                      const float *bias, int64_t B, int64_t H, int64_t L,
                      int64_t D, int64_t block, float cap, float *out,
                      float *lse, void *stream);

/*
 * ag_attn_fwd_strided_bias -- ag_attn_fwd with one bias per batch item.
 *
 * Each sequence has its own compact pair representation, hence its own bias
 * (page "Making Full-Context AlphaGenome Fit on an RTX 3090", section
 * "Profiling pointed at one very large object").  Batch item b reads
 * bias + b * bias_batch_stride, a [H, P, P] float32 block (P = ceil(L /
 * block)); bias_batch_stride is in floats, 0 (one bias shared by every item:
 * exactly ag_attn_fwd) or at least H * P * P (e.g. H * P * P for a dense
 * [B, H, P, P] tensor); anything else returns AG_ERR_SHAPE, as does a span
 * (B - 1) * bias_batch_stride + H * P * P above 2^56 floats.  Everything else
 * -- arguments, checks, results, scratch, stream behaviour -- as ag_attn_fwd.
 */
ag_status ag_attn_fwd_strided_bias(const void *q, const void *k, const void *v,
                                   const float *bias, int64_t bias_batch_stride,
                                   int64_t B, int64_t H, int64_t L, int64_t D,
                                   int64_t block, float cap, float *out,
                                   float *lse, void *stream);

/*
 * ag_attn_fwd_ex -- ag_attn_fwd_strided_bias with a value width Dv of its
 * own: v [B, L, Dv] and out [B, H, L, Dv].  The page's checkpoint has
 * Dv = 192 against D = 128 (section "Why stock FlashAttention was not a
 * drop-in replacement", tensors Q, K, V); the scale stays 1 / sqrt(D).
 * Supported: Dv == 128 or Dv == 192 (AG_ERR_UNSUPPORTED otherwise,
 * AG_ERR_SHAPE if Dv <= 0); v 16-byte aligned.  Everything else as
 * ag_attn_fwd_strided_bias, which is this call with Dv = D.
 */
ag_status ag_attn_fwd_ex(const void *q, const void *k, const void *v,
                         const float *bias, int64_t bias_batch_stride, int64_t B,
                         int64_t H, int64_t L, int64_t D, int64_t Dv, int64_t block,
                         float cap, float *out, float *lse, void *stream);

/*
 * ag_attn_fwd_query_slab -- ag_attn_fwd_ex for a slab of Lq consecutive query
 * positions of sequences of L positions (so that the queries can be split
 * between GPUs while every GPU holds all L keys and values: the sequence
 * parallelism of the page "From Code to Cure: How AlphaGenome Decodes the
 * 'Dark Matter' of DNA", section "The Architecture").
 *
 * Query i of this call is position q0 + i of its sequence for some q0 that
 * is a multiple of block (the caller's choice; the call never sees q0):
 *   q     [B, H, Lq, D]   the slab's queries
 *   k     [B, L, D], v [B, L, Dv]   all keys and values
 *   bias  [H, ceil(Lq / block), ceil(L / block)] per item: rows q0 / block ..
 *         of the full [H, P, P] bias (one per item at bias_batch_stride,
 *         0 or >= H * ceil(Lq / block) * ceil(L / block) floats)
 *   out   [B, H, Lq, Dv], lse [B, H, Lq]   the slab's results
 * Every query attends to all L keys, so the slab's rows equal the same rows
 * of a full call (bit for bit when both calls run those rows as whole pairs;
 * see ag_attn_fwd_schedule).  Lq == L with q0 = 0 is ag_attn_fwd_ex.
 * Checks and statuses as ag_attn_fwd_ex, plus AG_ERR_SHAPE for Lq < 0 and
 * AG_ERR_UNSUPPORTED for Lq > 65536; Lq == 0 is a no-op.
 */
ag_status ag_attn_fwd_query_slab(const void *q, const void *k, const void *v,
                                 const float *bias, int64_t bias_batch_stride, int64_t B,
                                 int64_t H, int64_t Lq, int64_t L, int64_t D, int64_t Dv,
                                 int64_t block, float cap, float *out, float *lse,
                                 void *stream);

/*
 * ag_attn_fwd_noalloc -- the attention forward on the range schedule, for
 * callers that cannot allocate device memory (the pages have no counterpart;
 * this is a library convenience).
 *
 * Same arguments, checks and stream behaviour as ag_attn_fwd, and the same
 * results within the tolerances of the forward (the schedule differs, so the
 * fp32 sums are grouped differently).  Its schedule cuts the (pair, key tile)
 * steps into equal contiguous runs, one per SM pair, and merges the pieces of
 * split pairs in a second kernel; those pieces need scratch, which here is a
 * static device array compiled into the library, 148 slots of 197,632 bytes
 * (29,249,536 bytes).  Callers for whom a library must not allocate: a
 * framework that has handed all device memory to its own pool, or a process
 * whose device memory budget is fixed at start-up.  The array is loaded with
 * the library's module for this entry point (lazy module loading: on the
 * first call) and stays on that GPU until the process exits.
 *
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current.
 *   - Returns AG_ERR_SCRATCH, launching nothing, when the call would use more
 *     than 148 slots (one per 2-CTA cluster of its grid: min(SM count / 2,
 *     work steps)), i.e. on a device with more than 296 SMs.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero.  Calls of this entry point that
 *     overlap on the GPU (two streams at once) race on it and must not be
 *     issued; calls of the other entry points do not touch it.
 */
ag_status ag_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                              const float *bias, int64_t B, int64_t H, int64_t L,
                              int64_t D, int64_t block, float cap, float *out,
                              float *lse, void *stream);

/*
 * ag_attn_fwd_launch_count -- how many kernels ag_attn_fwd (and
 * ag_attn_fwd_strided_bias, ag_attn_fwd_ex) launches for these sizes on the
 * current device: 0 for an empty call, 1, or 2 when some pairs of query tiles
 * have their keys split in two and a second launch merges them; for a cap
 * above 60 or no cap, the first pass of row maxima (1 or 2 launches) plus
 * the main kernel (a library convenience for callers that count launches;
 * the pages have no counterpart).  Same size and value checks, and
 * statuses, as ag_attn_fwd; count is a host pointer (AG_ERR_NULL if NULL).
 * Launches nothing.  The count is for value width D (128); at value width
 * 192 the caps above 60 run the running maximum, 1 or 2 launches.
 */
ag_status ag_attn_fwd_launch_count(int64_t B, int64_t H, int64_t L, int64_t D,
                                   int64_t block, float cap, int *count);

/*
 * ag_attn_fwd_schedule -- the work schedule of the attention forward for B
 * items of length L on a device with sm_pairs resident 2-CTA clusters (a
 * library convenience for inspecting and testing the host-side planner; the
 * pages have no counterpart).  Pure host logic: needs no GPU, launches
 * nothing.  Work unit: a "pair" is two 16-position query blocks of one item
 * (B * ceil(ceil(L/16)/2) pairs), each over n_kt = ceil(L/128) key tiles.
 *   with_scratch == 0 (ag_attn_fwd, _strided_bias, _ex): *sched = 1.  The
 *     first launch has *clusters clusters; cluster c runs whole pairs
 *     [wb[c], wb[c+1]) and then the first pieces (key tiles [0, *split_at))
 *     of split pairs [fb[c], fb[c+1]); split pair s is pair *n_whole + s.  If
 *     *tail_clusters > 0, a second launch has that many clusters and cluster
 *     c runs the second piece (key tiles [*split_at, n_kt)) of split pair c.
 *   with_scratch != 0 (ag_attn_fwd_noalloc's schedule): *sched = 0, the
 *     (pair, key tile) steps in *clusters equal contiguous runs (*whole = 1:
 *     rounded to whole pairs); wb, fb unused.
 * wb and fb are host arrays of 129 ints (written).  Statuses: AG_ERR_NULL
 * for a NULL pointer; the size checks of ag_attn_fwd (H = 8, D = 128,
 * block = 16); AG_ERR_SHAPE for B == 0, L == 0 or sm_pairs < 1.
 */
ag_status ag_attn_fwd_schedule(int64_t B, int64_t L, int sm_pairs, int with_scratch,
                               int *sched, int *clusters, int *tail_clusters, int *whole,
                               int *n_whole, int *split_at, int *wb, int *fb);

/*
 * ag_attn_bwd -- gradients of ag_attn_fwd_ex's out for an upstream gradient
 * dout: the chain rule through Eq. L_ij and the softmax (page "Making
 * Full-Context AlphaGenome Fit on an RTX 3090", section "Why stock
 * FlashAttention was not a drop-in replacement"; the page lists a backward
 * pass as later work for fine-tuning, section "Where I would take it next").
 * With x_ij the biased score, p_ij = exp(L_ij - lse_i) and
 * dp_ij = dout_i . v_j:
 *   delta_i = sum_j p_ij dp_ij,
 *   ds_ij   = p_ij (dp_ij - delta_i) (1 - tanh^2(x_ij / cap))  (no cap: 1),
 *   dq_i = sum_j ds_ij k_j / sqrt(D),  dk_j = sum_{h,i} ds_ij q_i / sqrt(D),
 *   dv_j = sum_{h,i} p_ij dout_i,  dbias cell = sum of ds_ij over the cell.
 *
 * Inputs (device, caller-owned, read only): q, k, v, bias,
 *   bias_batch_stride, B, H, L, D, Dv, block, cap exactly as
 *   ag_attn_fwd_ex; lse [B,H,L] float32 as written by the forward call on
 *   the same inputs; dout [B,H,L,Dv] float32.
 * Outputs (device, caller-owned, written, float32): dq [B,H,L,D],
 *   dk [B,L,D], dv [B,L,Dv] (K and V are shared by the heads, so their
 *   gradients sum over the heads), dbias in the layout of bias (with
 *   bias_batch_stride = 0 the one shared bias gets the sum over the items;
 *   otherwise item b's cells at dbias + b * bias_batch_stride, the padding
 *   between items untouched), delta [B,H,L].
 * Alignment: q, k, v 2 bytes, the float32 arrays 4 bytes; with Dv == 128
 *   also q, k, v, dout and dq 16 bytes (AG_ERR_ALIGN).  No output may
 *   overlap an input or another output (AG_ERR_ALIAS).  Size and value
 *   checks and their statuses as ag_attn_fwd_ex; B == 0 or L == 0 is a no-op.
 * Asynchronous on `stream`; no device memory is allocated; every output
 * value is written by one thread in a fixed order, so results are bitwise
 * reproducible.
 * Dv == 128 runs on the tensor cores (four kernels): dout is first split
 *   into two bf16 halves (hi = bf16(dout), lo = bf16(dout - hi)) stored in
 *   dq's memory (which the last kernel then overwrites with dq); the
 *   products with dout, P and dS take each as such a pair, so that they
 *   carry 16 significant bits, with fp32 accumulation.
 * Dv == 192 runs two float32 CUDA-core kernels.
 */
ag_status ag_attn_bwd(const void *q, const void *k, const void *v, const float *bias,
                      int64_t bias_batch_stride, const float *lse, const float *dout,
                      int64_t B, int64_t H, int64_t L, int64_t D, int64_t Dv,
                      int64_t block, float cap, float *dq, float *dk, float *dv,
                      float *dbias, float *delta, void *stream);

/*
 * ag_attn_bwd_launch_count -- how many kernels a non-empty ag_attn_bwd call
 * with value width Dv launches: 4 for Dv == 128, 2 for Dv == 192 (a library
 * convenience; the pages have no counterpart).  count is a host pointer
 * (AG_ERR_NULL if NULL); AG_ERR_SHAPE for Dv <= 0, AG_ERR_UNSUPPORTED for
 * other widths.  Launches nothing.
 */
ag_status ag_attn_bwd_launch_count(int64_t Dv, int *count);

/*
 * Device error word.  Every wait inside the kernels is bounded (about one
 * second); a wait that runs out makes the kernel stop, release what it
 * holds and record a code here instead of hanging the GPU.
 *   code == 0: no error.  Otherwise (site << 8) | kind, kind 1 = wait timeout.
 * ag_device_error synchronises `device`, copies the word of that device to
 * *code (host pointer) and clears it if `clear` != 0.  Returns AG_ERR_DEVICE
 * if the word was set, AG_OK if not, AG_ERR_CUDA/AG_ERR_NULL on failure.
 */
ag_status ag_device_error(int device, int *code, int clear);

/*
 * Self-test of the bounded waits: launches one block whose thread waits on an
 * mbarrier that nothing ever arrives at, for at most `timeout_ns`
 * nanoseconds (1 ms .. 10 s), and then records site 255 in the device error
 * word.  Lets a test check that a wait that runs out is reported and leaves
 * the context usable.  No fault and no hang: the wait is always bounded.
 */
ag_status ag_debug_wait_timeout(uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* AG_H_ */
