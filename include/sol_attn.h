/*
 * sol_attn.h -- C ABI of the Sol-Attn library (libsolattn.so, sm_100a).
 *
 * Sol-Attn is training-free, query-adaptive block-sparse attention.  The
 * pages that describe it give prose only; each entry point below names the
 * passage it implements:
 *
 *  [R1] "NVIDIA 团队开源 Sol-H3 的 DGX Spark 版本" (arex-research 3d0ff631),
 *       section "119.68 GiB memory pool", Sol-Attn bullet: blocks are picked
 *       during attention; each query block filters light query-key scores
 *       with its own threshold; selected blocks are exact; skipped blocks are
 *       corrected from pooled K/V summaries; routing, sparse compute and
 *       correction share one online softmax; no score map or routing index
 *       tensor is written; the operator is compared with FA4 (dense).
 *  [R2] Sol-H3 overview (yanziyuan 171844), "sparse attention" paragraph:
 *       64-token blocks; "safety rail" paragraph: the packed
 *       text | cond video | audio prefix always takes exact attention.
 *  [R3] "MiniMax 官宣 NVIDIA Sol 团队 H3 加速" (arex-research 2a2a70ca),
 *       section "speed-up comes from stacking every stage", Sol-Attn item:
 *       keep threshold = mean + tau x std of the query block's scores.
 *  [R4] "MiniMax 官推背书 Sol Engine" (arex-research 647c3193), section
 *       "3.95x near-lossless": skipped blocks get a Taylor-approximation
 *       compensation; this library implements its zeroth-order term
 *       (count-weighted mean-key logit + ln c_j, mean value).
 *  [R6] [R3]'s page, same section, fused-operators item: the QKNorm +
 *       partial RoPE chain keeps its intermediates in registers or on chip.
 *  [R7] [R1]'s page, section "latent hand-off: 384p draft to 768p refine":
 *       the DiT runs with 8-bit (W8A8 FP8) weights and activations; [R3]'s
 *       page, same section, multi-GPU item: attention outputs travel as FP8.
 *
 * Conventions shared by every entry point
 *  - q, k, v, out: DEVICE pointers to contiguous bf16 arrays laid out
 *    [B][H][N][D] (row-major, D fastest), 16-byte aligned, owned by the
 *    caller.  out must not overlap q, k, v or the workspace.
 *  - block must be 64; N and prefix_len must be multiples of 64; the
 *    prefix is tokens [0, prefix_len) of every (b, h) sequence.
 *  - D must be 64 or 128.  N / 64 must not exceed 4096 and B*H*N must fit
 *    in a signed 32-bit integer (SOL_ATTN_ERR_UNSUPPORTED otherwise).
 *  - B, H or N equal to 0 is an empty problem: SOL_ATTN_OK, nothing runs.
 *  - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous with respect to the host and issues no host
 *    synchronisation, except sol_attn_device_status(), and
 *    sol_attn_forward_host() on its error path or with a pageable `out`
 *    (see there).
 *  - Arguments are validated before any work is enqueued; a call that
 *    returns an error has enqueued nothing.  The library holds no state
 *    besides per-device cached attributes and one device error word.
 *  - Needs an sm_100 (B200-class) device: SOL_ATTN_ERR_ARCH otherwise.
 */
#ifndef SOL_ATTN_H
#define SOL_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SOL_ATTN_BLOCK 64

typedef enum {
  SOL_ATTN_OK = 0,
  SOL_ATTN_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment, prefix or tau */
  SOL_ATTN_ERR_UNSUPPORTED = 2,     /* valid but outside what the kernels cover */
  SOL_ATTN_ERR_ARCH = 3,            /* current device is not sm_100 */
  SOL_ATTN_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  SOL_ATTN_ERR_DEVICE_TIMEOUT = 5   /* a kernel wait gave up (see sol_attn_device_status) */
} sol_attn_status;

/* Optional extras of sol_attn_forward_ex / sol_attn_attend.  All pointers
 * are DEVICE pointers and may be NULL.  Zero-initialise unused fields. */
typedef struct {
  /* += number of (query block, key block) pairs kept exact, forced prefix
   * pairs included. */
  unsigned long long* kept_pairs;
  /* += number of (query block, key block) pairs the tensor cores computed
   * exactly: each 128-row tile visits the union of its two query blocks'
   * kept sets, so this is >= kept_pairs. */
  unsigned long long* exact_pairs;
  /* Keep bits for inspection, [B][H][M][ceil(M/32)] words, bit (j % 32) of
   * word (j / 32) of row (b, h, i) set iff key block j is kept for query
   * block i.  Only a debugging aid: when NULL (the normal case) no routing
   * data leaves the chip. */
  unsigned int* debug_mask;
  /* Softmax (and score) scale; 0 means 1 / sqrt(D).  Must be finite, >= 0. */
  float softmax_scale;
  /* Limit of every in-kernel wait, in milliseconds; 0 means 1000. */
  unsigned int timeout_ms;
  /* Test hook, keep 0: the loader skips the first key tile of every CTA so
   * the consumer's bounded wait runs out and the timeout path is exercised. */
  int test_skip_first_k_load;
  /* 0: routing by threshold (mean + tau * std).  > 0: fixed-budget routing of
   * the draft stage -- every video query block keeps its `budget_blocks`
   * highest-scoring video key blocks (same pooled scores; ties at the cut go
   * to the lower block index; tau is ignored), plus the prefix.  The draft
   * stage of the pages runs at 90 % video sparsity in 64-token blocks
   * (Sol-H3 DGX Spark release, section "latent hand-off: 384p draft to 768p
   * refine").  Must be >= 0. */
  int budget_blocks;
  /* Nonzero: skipped blocks are dropped instead of receiving the pooled
   * correction (plain block-sparse attention, as on the draft stage's
   * block-sparse backend). */
  int skip_correction;
} sol_attn_opts;

/* Sol-Attn forward [R1]-[R4]: pooling, routing, exact attention on kept
 * blocks, pooled correction of skipped blocks, one softmax.
 *   tau: threshold multiplier; -INFINITY keeps every block (dense result),
 *        +INFINITY keeps only the prefix; NaN is rejected.
 *   prefix_len: tokens of exact prefix (prefix query rows are dense and
 *        prefix key blocks are kept for every query block) [R2].
 * Per query block i >= P = prefix_len/64: s_ij = scale * <mean q, mean k_j>
 * over video key blocks j >= P; mu, sigma = population mean and std of
 * those scores; keep j iff s_ij >= mu + tau * sigma (all kept when the
 * scores are all equal).  A skipped block contributes logit
 * scale * <q_r, mean k_j> + ln 64 and value mean v_j.
 * Scratch: allocates sol_attn_workspace_bytes() with cudaMallocAsync on
 * `stream` and frees it with cudaFreeAsync on the same stream. */
int sol_attn_forward(const void* q, const void* k, const void* v, void* out, int B, int H,
                     int N, int D, int block, float tau, int prefix_len, void* stream);

/* Same as sol_attn_forward with the extras of `opts` (may be NULL). */
int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out, int B, int H,
                        int N, int D, int block, float tau, int prefix_len,
                        const sol_attn_opts* opts, void* stream);

/* Dense softmax attention softmax(q k^T / sqrt(D)) v: the comparator role of
 * FA4 in [R1], and the tau = -INFINITY limit of Sol-Attn.  Same layout
 * rules; needs no workspace and allocates nothing. */
int sol_attn_dense_forward(const void* q, const void* k, const void* v, void* out, int B,
                           int H, int N, int D, void* stream);

/* Bytes of scratch sol_attn_pool / sol_attn_attend need, and (if `offsets`
 * is not NULL) the byte offsets of its four sections, each 256-byte aligned,
 * with BHM = B*H*N/64 rows of D values:
 *   offsets[0] mean q   fp32 [BHM][D]
 *   offsets[1] mean k   fp32 [BHM][D]
 *   offsets[2] mean k   bf16 [BHM][D]  (round to nearest even of the fp32 mean)
 *   offsets[3] mean v   bf16 [BHM][D]
 * Returns 0 for invalid or empty shapes. */
size_t sol_attn_workspace_bytes(int B, int H, int N, int D, size_t* offsets);

/* Step 1 alone: block means of q, k, v [R1 "pooled K/V summaries", R2
 * 64-token blocks] into `workspace` (device, caller-owned, at least
 * sol_attn_workspace_bytes() bytes, 256-byte aligned). */
int sol_attn_pool(const void* q, const void* k, const void* v, void* workspace, int B, int H,
                  int N, int D, void* stream);

/* Steps 2-6 alone (routing, exact + pooled attention, epilogue) on a
 * workspace filled by sol_attn_pool for the same q, k, v.  `opts` may be
 * NULL. */
int sol_attn_attend(const void* q, const void* k, const void* v, void* out,
                    const void* workspace, int B, int H, int N, int D, int block, float tau,
                    int prefix_len, const sol_attn_opts* opts, void* stream);

/* Largest workspace sol_attn_forward_noalloc can serve: 64 MiB.  In whole
 * 64-token blocks that is B*H*(N/64) <= 43,690 at D = 128 (2,796,160 tokens)
 * and <= 87,381 at D = 64 (5,592,384 tokens; the workspace then fills the
 * array exactly). */
#define SOL_ATTN_NOALLOC_MAX_WORKSPACE (64u << 20)

/* Allocation-free variant of sol_attn_forward, for callers that cannot
 * allocate device memory while they run (a runtime that reserves all memory
 * up front, a server that must not enter the allocator between requests).
 * The paper has no counterpart; this is a deployment convenience.
 * Same arguments, layout and result as sol_attn_forward, but the pooled
 * workspace is a fixed array compiled into the library
 * (SOL_ATTN_NOALLOC_MAX_WORKSPACE bytes per device, held by every GPU that
 * loads the library until the process exits).  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *  - Shapes whose sol_attn_workspace_bytes() exceed the array return
 *    SOL_ATTN_ERR_UNSUPPORTED and enqueue nothing.
 *  - The first call on each device (with that device current) looks up the
 *    array's device address with cudaGetSymbolAddress.  Make that first
 *    call before any stream capture.
 *  - All calls share the one array.  Calls whose kernels overlap on the GPU
 *    (other streams, other host threads) race on it and must be serialised
 *    by the caller.  Nothing in it needs clearing: each call's pooling step
 *    overwrites every byte that its attention step reads. */
int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                             int H, int N, int D, int block, float tau, int prefix_len,
                             void* stream);

/* 8-bit variant of sol_attn_forward_ex [R1]-[R4], [R7]: q, k, v are DEVICE
 * arrays of E4M3 bytes (OCP FP8 E4M3: 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, largest finite 448), laid out [B][H][N][D] like the bf16
 * inputs, 16-byte aligned; the real values are the decoded bytes times
 * q_scale, k_scale, v_scale (finite, > 0; INVALID_ARG otherwise).  out is
 * bf16 [B][H][N][D] as elsewhere.  D must be 128 (UNSUPPORTED otherwise).
 * The operator is the same as sol_attn_forward's on the real values:
 *  - pooling and routing are computed in fp32 from the decoded values, so
 *    the keep mask follows the same definition;
 *  - the exact blocks and the pooled correction run on 8-bit tensor cores
 *    (fp32 accumulation): the pooled means used there are rounded to E4M3,
 *    and the probabilities P to E4M3 before the P V product.
 * Those two roundings are the only differences from the bf16 path's
 * arithmetic; the accuracy this gives is stated in the design notes.
 * `opts` (may be NULL) as in sol_attn_forward_ex.  Scratch, streams and
 * errors as in sol_attn_forward. */
int sol_attn_forward_fp8(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                         int D, int block, float tau, int prefix_len, float q_scale, float k_scale,
                         float v_scale, const sol_attn_opts* opts, void* stream);

/* sol_attn_forward_fp8's two steps alone, as sol_attn_pool / sol_attn_attend
 * are sol_attn_forward's: pooling of the E4M3 inputs into `workspace`
 * (sol_attn_workspace_bytes(B, H, N, 128) bytes, 256-byte aligned: the fp32
 * means of the real values for routing, and E4M3 means of the raw values in
 * the first half of the two 16-bit sections), then routing and attention on
 * that workspace.  Same argument rules as sol_attn_forward_fp8. */
int sol_attn_pool_fp8(const void* q, const void* k, const void* v, void* workspace, int B, int H, int N,
                      int D, float q_scale, float k_scale, void* stream);
int sol_attn_attend_fp8(const void* q, const void* k, const void* v, void* out, const void* workspace,
                        int B, int H, int N, int D, int block, float tau, int prefix_len, float q_scale,
                        float k_scale, float v_scale, const sol_attn_opts* opts, void* stream);

/* Host-buffer variant of sol_attn_forward: q, k, v and out are HOST
 * pointers, same [B][H][N][D] bf16 layout and the same result.  The pages
 * have no counterpart; this is the end-to-end path for a caller whose data
 * lives in host memory.
 * Every (b, h) sequence is an independent problem, so the B*H sequences are
 * cut into chunks of `heads_per_chunk` consecutive ones (0 picks about
 * 8 MiB of each tensor per chunk, at least one sequence and at most B*H; the
 * last chunk may be shorter).  Chunk c's host-to-device
 * copy runs on an internal copy stream while chunk c-1 is pooled and
 * attended on `stream` and chunk c-2 is copied back on a second internal
 * stream; three device buffer sets rotate.
 *  - Host memory should be page-locked (cudaHostAlloc or cudaHostRegister)
 *    for the copies to overlap the kernels; pageable memory gives the same
 *    result without the overlap.  With a pageable `out` the CUDA runtime
 *    makes each device-to-host copy return only once it has finished, so
 *    the call then blocks the host until the last chunk is back (an
 *    exception to the "no host synchronisation" rule above).
 *  - Device scratch: three chunk buffer sets of q, k, v, out plus one pooling
 *    workspace, allocated with cudaMallocAsync on `stream` and freed there.
 *  - The call returns once all work is enqueued; `out` is complete once
 *    `stream` has finished it.  The caller must keep the host buffers alive
 *    and unmodified until then.
 *  - Argument errors return before anything is enqueued; a CUDA error in
 *    the middle returns SOL_ATTN_ERR_CUDA and may leave earlier chunks
 *    enqueued (if their ordering before the scratch release cannot be
 *    enqueued either, the call synchronises its internal streams first).
 *    heads_per_chunk < 0 is SOL_ATTN_ERR_INVALID_ARG. */
int sol_attn_forward_host(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int N, int D, int block, float tau, int prefix_len, int heads_per_chunk,
                          void* stream);

/* QKNorm + partial RoPE of q and k, with the block pooling fused in [R6].
 * The pages name the chain only; this entry point fixes it as follows.
 * For every row x of q_in (and of k_in, with k_weight):
 *   y = x * rsqrt(mean(x^2) + eps) * q_weight          (RMSNorm over D)
 *   then for i < R/2, R = rope_dims, pos = token index in its sequence:
 *   (y_i, y_{i+R/2}) <- (y_i c - y_{i+R/2} s, y_i s + y_{i+R/2} c),
 *   c, s = cos, sin of pos * rope_base^(-2 i / R); dimensions >= R unchanged.
 * The results are written as bf16 to q_out and k_out.  If `workspace` is not
 * NULL, the same pass also fills it as sol_attn_pool(q_out, k_out, v) would,
 * bit for bit, so sol_attn_attend can follow without a separate pooling pass
 * over HBM; v is then required.  With workspace NULL only q_out and k_out are
 * written.
 *   q_weight, k_weight: DEVICE fp32 [D], 16-byte aligned.
 *   rope_dims: 0, or 16 * 2^k <= D (16, 32, 64 or 128).
 *   eps > 0 and finite; rope_base > 1 and finite.
 *   q_out and k_out must not overlap any input or each other.
 * Same shape rules as the other entry points; asynchronous on `stream`. */
int sol_attn_qknorm_rope_pool(const void* q_in, const void* k_in, const void* v, const float* q_weight,
                              const float* k_weight, void* q_out, void* k_out, void* workspace, int B, int H,
                              int N, int D, int rope_dims, float eps, float rope_base, void* stream);

/* Synchronises `stream`, then reads and clears the device error word that
 * kernels set when a bounded wait gives up.  SOL_ATTN_OK if none did,
 * SOL_ATTN_ERR_DEVICE_TIMEOUT if one did, SOL_ATTN_ERR_CUDA if the
 * synchronisation itself failed. */
int sol_attn_device_status(void* stream);

/* Static, human-readable name of a status code. */
const char* sol_attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H */
