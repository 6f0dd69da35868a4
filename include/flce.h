/*
 * flce.h — C ABI of libflce.so: the fused linear cross-entropy forward and
 * backward on NVIDIA B200 (sm_100a), with fp32, quantised-head,
 * host-input, vocabulary-parallel and no-allocation variants.
 *
 * The operation (D. Ineshin, "Een gefuseerde forward-kernel voor lineaire
 * cross-entropy op Apple-GPU's", 2026, section 1): for hidden states H (N, D),
 * an output projection W (V, D) and targets y (N),
 *     Z = H W^T,    loss_i = logsumexp(Z_i) - Z_{i, y_i},
 * computed by streaming vocabulary tiles through the online log-sum-exp
 *     m' = max(m, m_t),   s' = s * exp(m - m') + sum_j exp(z_j - m'),
 *     logsumexp = m + log(s) after the last tile,
 * and capturing the target logit in whichever tile holds it, so the (N, V)
 * logits matrix never exists (same section).  log is the natural logarithm.
 * The mean loss is the plain average of the N per-token losses.
 *
 * General contract of every entry point:
 *   - Pointers named H, W, y, out_*, workspace are DEVICE pointers on the
 *     current CUDA device, allocated and owned by the caller.  The library
 *     allocates no device or pinned memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; the call returns before the GPU finishes.
 *   - Host-detectable problems are returned synchronously and nothing is
 *     enqueued.  Problems found on the device (a target outside [0, V), a
 *     bounded wait that ran out) are recorded in the workspace status word
 *     and reported by flce_check().
 *   - Thread safety: calls on different workspaces may run concurrently.
 *     Calls that share one workspace must be ordered on one stream.
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLCE_API __attribute__((visibility("default")))
#else
#define FLCE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of H and W.  bf16 runs on the tcgen05 tensor-core path
 * (fp32 accumulation in TMEM).  fp32 inputs are first split, value by value,
 * into two bf16 parts hi = bf16(x), lo = bf16(x - hi) in the workspace, and
 * the same tensor-core path contracts hi*hi + hi*lo + lo*hi (three bf16
 * products per fp32 product, each accurate to about 3 * 2^-16 relative;
 * Henry, Tang and Heinecke, ARITH 2019).  fp32 values must be finite and
 * below bf16's largest finite value (about 3.39e38) in magnitude. */
typedef enum { FLCE_BF16 = 0, FLCE_FP32 = 1 } flce_dtype;

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_INVALID_ARG = 1,          /* null pointer, negative size, bad workspace, ... */
  FLCE_ERR_UNSUPPORTED = 2,          /* device is not sm_100, D % 8 != 0 or a pointer is
                                        not 16-byte aligned for bf16, sizes beyond int32 */
  FLCE_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < flce_workspace_size(...) */
  FLCE_ERR_CUDA = 4,                 /* a CUDA runtime/driver call or launch failed */
  FLCE_ERR_TARGET_OUT_OF_RANGE = 5,  /* (flce_check) some y_i outside [0, V) */
  FLCE_ERR_TIMEOUT = 6               /* (flce_check) a bounded device wait ran out */
} flce_status;

/* Schedule the library uses for one problem (host-side, informational).
 * The contraction is cut into work units of `block_rows` tokens by one vocab
 * slab; a slab is a run of consecutive `tile_cols`-column vocab tiles.  The
 * first `slab_rem` slabs hold slab_base + 1 tiles, the others slab_base. */
typedef struct {
  int64_t N, V, D;
  int32_t dtype;           /* flce_dtype */
  int32_t block_rows;      /* tokens per work unit (128 TMEM lanes per CTA) */
  int32_t tile_cols;       /* vocab columns per tile */
  int32_t k_block;         /* D elements per pipeline stage */
  int64_t token_blocks;    /* ceil(N / block_rows) */
  int64_t vocab_tiles;     /* ceil(V / tile_cols) */
  int32_t slabs;           /* P: partial (m, s) states per token */
  int32_t slab_base;       /* vocab_tiles / slabs */
  int32_t slab_rem;        /* vocab_tiles % slabs */
  int32_t grid;            /* CTAs launched for the contraction kernel */
  int64_t units;           /* token_blocks * slabs */
  int64_t makespan_tiles;  /* tiles processed by the busiest CTA (or CTA pair) */
  size_t workspace_bytes;  /* == flce_workspace_size(N, V, D, dtype) */
  int32_t ctas_per_unit;   /* 2: a CTA pair shares each 256-token tile (N > 128);
                              1: one CTA per tile */
  int32_t group_blocks;    /* token blocks per raster group: units are ordered group by
                              group, slab-major inside a group, and handed out round-robin */
} flce_plan_t;

/* Bytes of device workspace that flce_forward / flce_partials need for this
 * problem: a 256-byte header, one 4-byte arrival counter per 128 tokens, the
 * per-(slab, token) partial states (8 bytes each, at most 512 slabs per
 * token, so O(N), never O(N*V)), and one fp64 per 128 tokens for the mean.  fp32 inputs add the bf16 split copies of H
 * and W ([hi | lo], 4 Dp bytes per row each), Dp = D rounded up to 64:
 * O((N + V) D), still never O(N*V).  Depends only on its arguments (not on
 * the device).
 * Returns 0 for invalid arguments (N < 0, V < 1, D < 1, unknown dtype).  Host
 * only; never touches the GPU. */
FLCE_API size_t flce_workspace_size(int64_t N, int64_t V, int64_t D, flce_dtype dtype);

/* The schedule for a device with `sm_count` SMs, assuming every SM pair can
 * hold a CTA pair (host only, no GPU call; at launch the library sizes the
 * grid from the device's actual cluster occupancy).
 * Returns FLCE_ERR_INVALID_ARG for invalid sizes, sm_count < 1 or plan NULL. */
FLCE_API flce_status flce_plan(int64_t N, int64_t V, int64_t D, flce_dtype dtype, int32_t sm_count,
                      flce_plan_t* plan);

/* The partition-aware order of the pair kernel's work units (host only, no
 * GPU call).  B200's L2 is two partitions, each caching what its own SMs
 * read.  When a forward has at least 16 units per CTA pair and more token
 * blocks than one raster group (flce_plan_t group_blocks), the pairs on
 * partition 0 take the first side0_units units of the token-block-major
 * order and the pairs on partition 1 the rest, each side slab-major over its
 * own token blocks (the units and their arithmetic are those of the plain
 * order; only which pair computes which unit changes, so results are bitwise
 * the same).  The first such forward on a device maps the partitions with two
 * small kernels on the caller's stream and waits for them (once per device;
 * not while the stream is being captured into a CUDA graph, where the plain
 * order is used until a forward runs outside a capture).
 *
 * flce_partition_order writes, for token_blocks TB and slabs P, the (slab,
 * token block) of each unit of partition 0's list and then of partition 1's:
 * 2 TB P int32 values to out.  FLCE_ERR_INVALID_ARG if TB < 1, P < 1,
 * TB P >= 2^30, side0_units outside [0, TB P] or out NULL.
 *
 * flce_partition_take: the (partition, rank) a pair takes when it arrives as
 * number `arrival` (from 0) on partition `side`, with pairs0 and pairs1 pairs
 * planned on the two partitions and pairs0 + pairs1 pairs launched: its own
 * rank while the side has fewer than planned, else the highest rank of the
 * other side that no pair of that side can reach.  FLCE_ERR_INVALID_ARG if a
 * count is < 1, side is not 0 or 1, arrival is outside [0, pairs0 + pairs1)
 * or an output is NULL. */
FLCE_API flce_status flce_partition_order(int32_t token_blocks, int32_t slabs,
                                          int32_t side0_units, int32_t* out);
FLCE_API flce_status flce_partition_take(int32_t pairs0, int32_t pairs1, int32_t side,
                                         int32_t arrival, int32_t* out_side, int32_t* out_rank);

/* The current device's partition map, if a forward has taken it: the CTA
 * pairs found resident on partitions 0 and 1 (out_pairs[2]).  Returns
 * FLCE_ERR_UNSUPPORTED while there is none (no forward large enough has run
 * on the device, or the latencies did not split into two clear groups, in
 * which case every forward uses the plain order), FLCE_ERR_INVALID_ARG for a
 * NULL pointer.  Host only: reads what the library recorded. */
FLCE_API flce_status flce_partition_map(int32_t* out_pairs);

/*
 * The full forward: per-token loss, log-sum-exp and target logit, and the
 * mean loss.  Section 1 of the page: loss_i = logsumexp(Z_i) - Z_{i, y_i}.
 *
 *   H            (N, D) row-major, dtype elements, contiguous (row stride D)
 *   W            (V, D) row-major, dtype elements, contiguous (row stride D)
 *   y            (N) int64 targets; each must lie in [0, V)
 *   N >= 0, V >= 1, D >= 1; N, V < 2^31.  bf16 also needs D % 8 == 0 and
 *                16-byte-aligned H and W (tensor-memory-access strides).
 *   out_loss, out_lse, out_target_logit   (N) fp32 each, written for every row
 *   out_mean     (1) fp32 or NULL; mean of out_loss computed in fp64
 *   workspace    >= flce_workspace_size(N, V, D, dtype) bytes, 256-byte aligned;
 *                contents on entry are ignored; it holds the status word that
 *                flce_check() reads until the next call that uses it
 *   stream       cudaStream_t
 * One contraction launch, after a kernel that clears the workspace header:
 * a one-block clear that the contraction overlaps (programmatic stream
 * serialization), or for fp32 inputs the split of H and W and for N < 32 the
 * padded copy of H, which clear it in their first block.  The CTA that writes
 * the last vocab slab's state of a 128-token row block merges that block in
 * the same kernel, and the one that merges the last row block forms the mean.
 * The results equal those of flce_partials followed by flce_merge bit for bit.
 * A row whose target is out of range gets NaN loss and NaN target logit and
 * sets FLCE_ERR_TARGET_OUT_OF_RANGE for flce_check().  N == 0 is a no-op that
 * returns FLCE_OK and writes nothing (out_mean untouched).
 * Results are bitwise deterministic run to run on the same device.
 */
FLCE_API flce_status flce_forward(const void* H, const void* W, const int64_t* y,
                         int64_t N, int64_t V, int64_t D, flce_dtype dtype,
                         float* out_loss, float* out_lse, float* out_target_logit,
                         float* out_mean, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Element type of the targets y in flce_forward_ex. */
typedef enum { FLCE_INDEX_INT64 = 0, FLCE_INDEX_INT32 = 1 } flce_index_dtype;

/* Arguments of flce_forward_ex: those of flce_forward plus row strides, the
 * target type and an optional sum of the losses. */
typedef struct {
  const void* H;            /* (N, D) rows, row stride ldh elements */
  int64_t ldh;              /* >= D; 0 means D.  bf16: a multiple of 8 */
  const void* W;            /* (V, D) rows, row stride ldw elements */
  int64_t ldw;              /* >= D; 0 means D.  bf16: a multiple of 8 */
  const void* y;            /* (N) targets of type y_dtype, each in [0, V) */
  int32_t y_dtype;          /* flce_index_dtype */
  int32_t dtype;            /* flce_dtype of H and W */
  int64_t N, V, D;
  float* out_loss;          /* (N) */
  float* out_lse;           /* (N) */
  float* out_target_logit;  /* (N) */
  float* out_mean;          /* (1) or NULL */
  float* out_sum;           /* (1) or NULL: sum_i out_loss[i], the fp64 total that the
                               mean divides by N, rounded once to fp32 */
} flce_forward_args;

/*
 * flce_forward with strided H and W (for example slices of larger buffers)
 * and int32 or int64 targets.  Same operation, workspace (sized by
 * flce_workspace_size(N, V, D, dtype)), results and error behaviour as
 * flce_forward; FLCE_ERR_INVALID_ARG for a bad stride or index type,
 * FLCE_ERR_UNSUPPORTED for a bf16 stride that is not a multiple of 8.
 */
FLCE_API flce_status flce_forward_ex(const flce_forward_args* args, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * First stage of flce_forward, on its own: the contraction Z = H W^T tile by
 * tile with the online (m, s) update of section 1 of the page, leaving one
 * partial state per (vocab slab, token) in the workspace and writing the
 * target logit of every row whose target is in range (from the tile that
 * holds it).  Arguments as for flce_forward.  Resets the workspace status
 * word.  Must be followed by flce_merge on the same workspace and stream.
 */
FLCE_API flce_status flce_partials(const void* H, const void* W, const int64_t* y,
                          int64_t N, int64_t V, int64_t D, flce_dtype dtype,
                          float* out_target_logit, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Second stage: combines the partial states left by flce_partials in a fixed
 * order (m = max_p m_p, s = sum_p s_p exp(m_p - m), logsumexp = m + log s:
 * the same recurrence applied to whole slabs), then writes loss = lse -
 * target logit, and the mean if out_mean is not NULL.  N, V and y must be
 * those given to flce_partials; out_target_logit is read (and set to NaN for
 * out-of-range targets).
 */
FLCE_API flce_status flce_merge(const int64_t* y, int64_t N, int64_t V,
                       float* out_loss, float* out_lse, float* out_target_logit,
                       float* out_mean, const void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * Backward of the weighted loss sum_i g_i loss_i (g_i = grad_scale *
 * grad_loss[i], or grad_scale when grad_loss is NULL; g_i = 1/N for the mean
 * loss).  Differentiating section 1 of the page:
 *     dZ_ij = g_i (exp(z_ij - lse_i) - [j == y_i]),   dH = dZ W,   dW = dZ^T H.
 * As on the page, the forward's log-sum-exp is kept and the logits are
 * regenerated tile by tile; vocabulary chunks (32768 rows for bf16, 16384 for
 * fp32) bound the working slice of dZ to O(N * chunk) (never O(N * V)).
 *
 *   H, W, y, N, V, D, dtype   as for flce_forward (bf16: D % 8 == 0 and
 *                             16-byte-aligned H, W; fp32: any D, 4-byte
 *                             alignment)
 *   lse          (N) fp32: out_lse of the forward on the same H, W
 *   grad_loss    (N) fp32 upstream gradient dL/dloss_i, or NULL
 *   dH           (N, D) fp32 row-major, overwritten
 *   dW           (V, D) fp32 row-major, overwritten
 *   workspace    >= flce_backward_workspace_size(N, V, D, dtype) bytes,
 *                256-byte aligned (the status word read by flce_check and one
 *                N x chunk slice of dZ in bf16: 256 B + 2 N chunk B, chunk =
 *                min(V rounded up to 256, 32768 (bf16) or 16384 (fp32)),
 *                each part rounded up to
 *                256 B; fp32 inputs add a second dZ slice and the bf16
 *                hi/lo split copies of H and of one W chunk, 6 Dp bytes per
 *                row, Dp = D rounded up to 8)
 * bf16 inputs: dZ is rounded to bf16 before the two gradient contractions
 * (fp32 accumulation), so each gradient entry carries an error of at most
 * about 2^-8 times sum_j |dZ_ij| |W_jk| (resp. sum_i |dZ_ij| |H_ik|).
 * fp32 inputs: H, W and dZ are each carried as two bf16 parts (hi + lo, to
 * 2^-16 relative) and every contraction runs the three products hi*hi +
 * hi*lo + lo*hi, about 3 * 2^-16 of the same magnitudes.
 * A target outside [0, V) sets FLCE_ERR_TARGET_OUT_OF_RANGE for flce_check.
 * Deterministic run to run.
 */
FLCE_API size_t flce_backward_workspace_size(int64_t N, int64_t V, int64_t D, flce_dtype dtype);

FLCE_API flce_status flce_backward(const void* H, const void* W, const int64_t* y,
                                   const float* lse, const float* grad_loss, float grad_scale,
                                   int64_t N, int64_t V, int64_t D, flce_dtype dtype, float* dH,
                                   float* dW, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Vocabulary-parallel forward (W split by rows over G ranks or devices).
 * The recurrence of section 1 of the page is associative over any split of
 * the vocabulary, so each shard can fold its own columns and the shards'
 * states merge exactly like the tiles of one device:
 *   1. each shard r: flce_partials_shard on its rows W[v_offset, v_offset + V_shard)
 *      (y holds global vocabulary ids), then flce_shard_state -> one
 *      {m, s, target logit, owned} float4 per token;
 *   2. gather the G state arrays in shard order (e.g. one all-gather of
 *      16 N bytes per rank);
 *   3. flce_merge_shards -> loss, lse, target logit and mean for the whole
 *      vocabulary.
 * Workspaces and scratch are caller-owned device memory, as elsewhere.
 */

/* flce_partials on the vocabulary shard W_shard = W[v_offset, v_offset +
 * V_shard): writes the target logit only for rows whose target lies in the
 * shard; other rows of out_target_logit are left as they were.  Sizes and
 * workspace as for flce_partials with V = V_shard; v_offset >= 0. */
FLCE_API flce_status flce_partials_shard(const void* H, const void* W_shard, const int64_t* y,
                                         int64_t N, int64_t V_shard, int64_t v_offset, int64_t D,
                                         flce_dtype dtype, float* out_target_logit, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* After flce_partials_shard on `workspace`: out_state (N float4, 16-byte
 * aligned) = {m, s, target logit, owned} per token, where (m, s) folds the
 * shard's slab states and owned = 1 iff v_offset <= y_i < v_offset + V_shard
 * (target is then the shard's target logit, else 0). */
FLCE_API flce_status flce_shard_state(const int64_t* y, int64_t N, int64_t V_shard,
                                      int64_t v_offset, const float* target_logit,
                                      const void* workspace, size_t workspace_bytes,
                                      float* out_state, void* stream);

/* Bytes of scratch flce_merge_shards needs: 256 + 8 ceil(N / 256), rounded. */
FLCE_API size_t flce_merge_shards_scratch_size(int64_t N);

/* Merges G shard states, laid out [G][N] float4 in shard order (any order
 * gives the same lse up to rounding; a fixed order makes it deterministic),
 * into per-token loss, lse and target logit, the mean (out_mean may be
 * NULL) and the sum of the losses (out_sum may be NULL; the fp64 total that
 * the mean divides by N, rounded once).  A token whose target is outside [0, V_total) or is held by no
 * shard or by more than one gets NaN and sets FLCE_ERR_TARGET_OUT_OF_RANGE
 * in the scratch status word (read with flce_check(scratch, stream)). */
FLCE_API flce_status flce_merge_shards(const float* states, int32_t G, const int64_t* y, int64_t N,
                                       int64_t V_total, float* out_loss, float* out_lse,
                                       float* out_target_logit, float* out_mean, float* out_sum,
                                       void* scratch, size_t scratch_bytes, void* stream);

/* Waits for `stream`, then reads the workspace status word left by the last
 * flce_forward / flce_partials + flce_merge that used this workspace.
 * Returns FLCE_OK, FLCE_ERR_TARGET_OUT_OF_RANGE, FLCE_ERR_TIMEOUT,
 * FLCE_ERR_INVALID_ARG (merge saw a workspace flce_partials did not prepare)
 * or FLCE_ERR_CUDA. */
FLCE_API flce_status flce_check(const void* workspace, void* stream);

/* Static, NUL-terminated description of a status code (never NULL). */
FLCE_API const char* flce_status_string(flce_status status);

/*
 * Self-test of the bounded device waits.  Launches one CTA whose thread
 * waits on a shared-memory barrier that nothing completes, with a limit of
 * `limit_ns` nanoseconds (1000 <= limit_ns <= 10^9); the wait gives up,
 * records FLCE_ERR_TIMEOUT in the workspace status word and the kernel
 * returns normally.  `workspace` needs 256 bytes.  Use flce_check() to read
 * the result.  No GPU fault, trap or hang is involved.
 */
FLCE_API flce_status flce_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                       uint64_t limit_ns, void* stream);

/*
 * flce_forward without a caller-supplied workspace, for callers that cannot
 * allocate device memory when they need the loss: code that runs inside an
 * allocator or memory-pool callback, runtimes that forbid cudaMalloc while
 * they own the device memory budget, or hosts with no spare buffer to pass.
 * The page has no counterpart to this entry point; it only changes where the
 * workspace lives.
 *
 * The scratch is a fixed device array of FLCE_NOALLOC_SCRATCH_BYTES (64 MiB)
 * inside the library's CUDA module.  Every GPU on which the library's kernels
 * are loaded holds it until the process exits.  The call allocates nothing:
 * no cudaMalloc, cudaFree or allocating library routine.
 *   - Arguments, results and errors are those of flce_forward, except that
 *     there is no workspace argument.
 *   - A problem whose flce_workspace_size(N, V, D, dtype) exceeds
 *     FLCE_NOALLOC_SCRATCH_BYTES is rejected with FLCE_ERR_WORKSPACE_TOO_SMALL
 *     and nothing is enqueued.  With V >= 131072 (512 slab states per token)
 *     that means N <= 16383.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current.  Make that first call
 *     before any stream capture on that device.  The address is cached with
 *     the id of the CUDA context it belongs to; a call in another context
 *     (a non-primary context, or the primary context re-created after
 *     cudaDeviceReset) looks it up again, so it too should come before any
 *     capture in that context.
 *   - All calls on one device share the array, and it keeps the contents of
 *     the last call.  Each call resets the header words it needs before its
 *     kernels run.  Calls whose work overlaps on the GPU (different streams,
 *     or threads without ordering) race on the array and give wrong results:
 *     order them on one stream.
 *   - The device status word lives in the shared array, so flce_check() does
 *     not apply.  An out-of-range target still gives a NaN loss and target
 *     logit for its row.
 */
#define FLCE_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

FLCE_API flce_status flce_forward_noalloc(const void* H, const void* W, const int64_t* y,
                                          int64_t N, int64_t V, int64_t D, flce_dtype dtype,
                                          float* out_loss, float* out_lse, float* out_target_logit,
                                          float* out_mean, void* stream);

/*
 * Quantised output head.
 *
 * The page (section 2) says its first, pure-MLX prototype supported dense and
 * quantised output heads; it does not define the quantised format, and its
 * measurements leave the quantised variants out (section 9).  Format read
 * here: MLX's affine group quantisation.  Each row j of W (V, D) is cut into
 * groups of G consecutive elements along D; group g of row j has a bf16 scale
 * s_jg and a bf16 bias b_jg, and element k holds an unsigned `bits`-bit code
 * q_jk, so that
 *     W_jk = s_{j, k/G} * q_jk + b_{j, k/G}.
 * The loss is the section-1 operation on that W.
 *
 *   H        (N, D) bf16, contiguous, 16-byte aligned
 *   wq       (V, D * bits / 32) uint32, contiguous, 16-byte aligned: the codes
 *            of a row packed 32 / bits per word, lowest bits first (element k
 *            in word k / (32/bits) at bit offset bits * (k mod (32/bits)))
 *   scales, biases   (V, D / G) bf16 each, contiguous
 *   bits     2, 4 or 8;  group_size G: 32, 64 or 128;  D a multiple of G
 *   y, N, V, D, out_*      as flce_forward (int64 targets); out_sum (1) fp32 or
 *            NULL receives the sum of the losses (the fp64 total that the
 *            mean divides by N, rounded once)
 *   workspace  >= flce_quantized_workspace_size(N, V, D, bits, group_size)
 *            bytes, 256-byte aligned; holds the status word flce_check() reads
 *
 * How it runs: W is expanded 16384 vocabulary rows at a time into the
 * workspace as two bf16 K segments per row, hi = bf16(W_jk) and lo =
 * bf16(W_jk - hi) (W_jk formed in fp32 with one rounding), and the
 * tensor-core contraction stages each K block of H once with both parts of
 * W and forms H hi^T + H lo^T: twice the tensor work of a bf16 head, with
 * |W - hi - lo| <= 2^-16 |W| per weight.  Each chunk is a
 * vocabulary shard; their per-token states are merged at the end, in chunk
 * order.  The workspace is O(N V / 16384 + 16384 D), never O(N V).
 * Errors: FLCE_ERR_INVALID_ARG for bad sizes, formats, null pointers or a
 * misaligned workspace / scales / biases; FLCE_ERR_UNSUPPORTED for a
 * misaligned H or wq, sizes beyond int32 or a device that is not sm_100;
 * FLCE_ERR_WORKSPACE_TOO_SMALL.  Targets are checked on the device as in
 * flce_forward.  N == 0 is a no-op that returns FLCE_OK.
 */
FLCE_API size_t flce_quantized_workspace_size(int64_t N, int64_t V, int64_t D, int32_t bits,
                                              int32_t group_size);

FLCE_API flce_status flce_forward_quantized(const void* H, const uint32_t* wq,
                                            const void* scales, const void* biases,
                                            int32_t bits, int32_t group_size, const int64_t* y,
                                            int64_t N, int64_t V, int64_t D, float* out_loss,
                                            float* out_lse, float* out_target_logit,
                                            float* out_mean, float* out_sum, void* workspace,
                                            size_t workspace_bytes, void* stream);

/*
 * Vocabulary-parallel backward: this caller holds W rows [v_offset, v_offset
 * + V_shard) of a V_total-word vocabulary (as in flce_partials_shard).  With
 * lse the log-sum-exp over the WHOLE vocabulary (flce_merge_shards), it
 * writes this shard's rows of dW and this shard's share of dH:
 *     dH_partial = sum_{j in shard} dZ_ij W_j,     dW_shard = dZ_shard^T H,
 * so that dH is the sum of dH_partial over the shards (one all-reduce; the
 * Python binding's backward_vocab_parallel does it over torch.distributed).
 * A target outside the shard adds no one-hot term here; a target outside
 * [0, V_total) sets FLCE_ERR_TARGET_OUT_OF_RANGE.  Arguments, workspace
 * (flce_backward_workspace_size(N, V_shard, D, dtype)), precision and errors
 * otherwise as flce_backward; FLCE_ERR_INVALID_ARG if the shard does not lie
 * inside [0, V_total).
 *   dh_ready_event  a cudaEvent_t or NULL: recorded on `stream` as soon as
 *            dH_partial is final, before the last chunk's dW GEMMs, so that a
 *            collective on dH (on another stream waiting for the event) can
 *            overlap them.
 */
FLCE_API flce_status flce_backward_shard(const void* H, const void* W_shard, const int64_t* y,
                                         const float* lse, const float* grad_loss,
                                         float grad_scale, int64_t N, int64_t V_shard,
                                         int64_t v_offset, int64_t V_total, int64_t D,
                                         flce_dtype dtype, float* dH_partial, float* dW_shard,
                                         void* workspace, size_t workspace_bytes, void* stream,
                                         void* dh_ready_event);

/*
 * Backward of the forward with a quantised head: dH only.  A quantised head
 * is frozen while the rest of the model trains (its codes cannot take a
 * gradient step), so only the hidden-state gradient is formed:
 *     dZ_ij = g_i (exp(z_ij - lse_i) - [j == y_i]),   dH = dZ W,
 * with W the dequantised head (same format and arguments as
 * flce_forward_quantized), g_i and lse as in flce_backward.
 *   dH         (N, D) fp32 row-major, overwritten
 *   workspace  >= flce_backward_quantized_workspace_size(N, V, D, bits,
 *              group_size) bytes, 256-byte aligned: the status word, an
 *              N x chunk bf16 slice of dZ and one chunk of W expanded to bf16
 *              [hi | lo] (chunks of 16384 vocabulary rows)
 * Per chunk: the codes are expanded as in flce_forward_quantized, the logits
 * regenerated as [H | H] [hi | lo]^T on the tensor cores, dZ rounded to bf16,
 * and dH accumulates dZ W_hi + dZ W_lo in that order: each entry is within
 * about 2^-8 sum_j |dZ_ij| |W_jk| of the exact value (as flce_backward on
 * bf16 inputs).  Errors as flce_forward_quantized; targets are checked on the
 * device.  Deterministic.  N == 0 is a no-op.
 */
FLCE_API size_t flce_backward_quantized_workspace_size(int64_t N, int64_t V, int64_t D,
                                                       int32_t bits, int32_t group_size);

FLCE_API flce_status flce_backward_quantized(const void* H, const uint32_t* wq,
                                             const void* scales, const void* biases,
                                             int32_t bits, int32_t group_size, const int64_t* y,
                                             const float* lse, const float* grad_loss,
                                             float grad_scale, int64_t N, int64_t V, int64_t D,
                                             float* dH, void* workspace, size_t workspace_bytes,
                                             void* stream);

/*
 * The forward on inputs that live in HOST memory, results returned to host
 * memory: the same operation as flce_forward (section 1 of the page), for
 * callers whose H, W and y are not on the device (W offloaded to the host,
 * data loaders that produce pinned host batches).
 *
 *   H_host (N, D) bf16, W_host (V, D) bf16, y_host (N) int64: host memory,
 *            contiguous.  Page-locked (pinned) memory lets the copies run
 *            asynchronously and overlap the contraction; pageable memory
 *            works but the copies then block the calling thread.  The host
 *            buffers must stay valid and unchanged until `stream` has been
 *            synchronised.
 *   loss_host (N) fp32 host buffer (required); lse_host, target_logit_host
 *            (N) and mean_host (1) may be NULL.  They are written by copies
 *            enqueued on `stream`: read them after synchronising `stream`.
 *   N, V, D  as flce_forward; bf16 only (fp32 returns FLCE_ERR_UNSUPPORTED),
 *            D % 8 == 0.
 *   workspace  device memory, >= flce_forward_host_workspace_size(N, V, D,
 *            dtype) bytes, 256-byte aligned: device copies of H and y, the
 *            outputs, two staging buffers of 8192 W rows, and the merge
 *            state; holds the status word flce_check() reads.
 *   stream   cudaStream_t for the kernels and the result copies.
 *   copy_stream  cudaStream_t for the host-to-device copies (a different
 *            stream overlaps them with the kernels); NULL = use `stream`.
 *
 * W crosses PCIe in chunks of 8192 rows into two alternating staging
 * buffers; each chunk's contraction (a vocabulary shard) starts as soon as
 * its copy lands and runs while the next chunk is copied, and the chunks'
 * per-token states are merged in chunk order at the end.  The call first
 * makes copy_stream wait for the work already queued on `stream`, so calls
 * on one (stream, workspace) pair may be issued back to back.  The library
 * creates and destroys a few CUDA events per call and allocates no memory.
 * Errors as flce_forward; targets are checked on the device.  N == 0 is a
 * no-op.
 */
FLCE_API size_t flce_forward_host_workspace_size(int64_t N, int64_t V, int64_t D,
                                                 flce_dtype dtype);

FLCE_API flce_status flce_forward_host(const void* H_host, const void* W_host,
                                       const int64_t* y_host, int64_t N, int64_t V, int64_t D,
                                       flce_dtype dtype, float* loss_host, float* lse_host,
                                       float* target_logit_host, float* mean_host,
                                       void* workspace, size_t workspace_bytes, void* stream,
                                       void* copy_stream);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H_ */
