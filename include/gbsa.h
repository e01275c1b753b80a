/*
 * gbsa.h -- C ABI of libgbsa: block-sparse flash attention over a paged KV
 * cache with grouped-query heads (forward pass), for NVIDIA B200 (sm_100a).
 *
 * Source of the operation: the GenericBlockSparseAttention article
 * (cf-1.com/news/4865651, "GBSA article" below) and the FlashAttention blog
 * post on CANN ops-transformer (ai6s.net, "FA blog" below).
 *
 *   out = Softmax(scale * Q * K_sparse^T + mask) * V_sparse
 *       (GBSA article, "Function / sparse attention mechanism", the formula)
 *
 * Q is cut into blocks of block_x query tokens; every Q block, per KV head,
 * attends only to the sparse_count[kvh][qb] KV blocks listed in
 * sparse_idx[kvh][qb][0:top_k].  A KV block is one 128-token page of the
 * paged K/V pool, found through block_table (layout PA_BBND).  The scores are
 * computed tile by tile with an online softmax (FA blog, "three steps"), so
 * the score matrix never exists; the log-sum-exp can be written out.
 *
 * Two-phase use, as in the GBSA article ("two-phase call: metadata first"):
 *   1. gbsa_metadata()  builds the load-balanced work list on the device;
 *   2. gbsa_forward()   runs the attention from that work list.
 * The metadata must be rebuilt for every call whose index/count/length
 * tensors change, with the same problem description as the forward call.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory, never synchronises the stream and
 *     never reads device values on the host.  Work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - Host-detectable rule violations return a non-zero gbsa_status before
 *     anything is launched.  Values inside device tensors are not checked on
 *     the host (GBSA article, "Constraints": tiling does not check values);
 *     when `dev_status` is non-NULL the kernels OR GBSA_DEV_* bits into that
 *     device int32 instead (and skip the offending work; they never trap).
 *   - Every kernel after the first of a call is launched with programmatic
 *     stream serialization: it may start while the previous kernel on the
 *     stream is finishing, and waits for that kernel's completion before it
 *     reads or writes global memory, so stream order holds as usual.
 *   - Layouts (GBSA article, "Parameters" and the aclnn example call); the
 *     element type of q, k and v is gbsa_problem.dtype (bf16, fp16 or E4M3):
 *       q            [T, N1, D]                 contiguous   (TND)
 *       k, v         [num_pages, 128, N2, D]    only dim0 may be strided:
 *                    stride0 = kv_page_stride elements  (PA_BBND), or
 *                    [T_kv, N2, D] contiguous with cu_seqlens_kv (TND)
 *       sparse_idx   [N2, total_q_blocks, top_k] int32, contiguous
 *       sparse_count [N2, total_q_blocks]        int32, contiguous
 *       cu_seqlens_q [B+1]                       int64 prefix sums of the
 *                                                Q storage lengths
 *       seqused_q    [B] int32 (optional), seqused_kv [B] int32 (required)
 *       block_table  [B, max_pages_per_seq]      int32 logical->physical page
 *       out          [T, N1, D] fp16 for fp16 inputs, else bf16;
 *       lse          [T, N1] fp32 (natural log)
 */
#ifndef GBSA_H
#define GBSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GBSA_ABI_VERSION 6

/* Symbols of the C ABI are exported; everything else in libgbsa is hidden. */
#if defined(__GNUC__)
#define GBSA_API __attribute__((visibility("default")))
#else
#define GBSA_API
#endif

/* Return codes.  The GBSA article's return-code table did not survive
 * extraction; these are this library's own. */
typedef enum gbsa_status {
  GBSA_OK = 0,
  GBSA_ERR_INVALID_ARG = 1,         /* NULL pointer, negative size, bad enum value     */
  GBSA_ERR_UNSUPPORTED = 2,         /* a mode the article lists as unsupported         */
  GBSA_ERR_SHAPE = 3,               /* a dimension rule of "Constraints" is violated   */
  GBSA_ERR_ALIGNMENT = 4,           /* a pointer or stride is not 16-byte aligned      */
  GBSA_ERR_WORKSPACE_TOO_SMALL = 5, /* workspace smaller than gbsa_workspace_size()    */
  GBSA_ERR_METADATA_TOO_SMALL = 6,  /* metadata smaller than gbsa_metadata_size()      */
  GBSA_ERR_CUDA = 7,                /* a CUDA runtime/driver call failed               */
  GBSA_ERR_NO_DEVICE = 8            /* num_ctas = 0 needs a device, and none is usable */
} gbsa_status;

/* Bits OR-ed into *dev_status by the kernels (device-side validation). */
#define GBSA_DEV_BAD_SEQLEN 0x01      /* cu_seqlens_q not monotone / not ending at T, seqused_q > storage,
                                         seqused_kv < 0, or the Q blocks do not add up to total_q_blocks */
#define GBSA_DEV_BAD_BLOCK_IDX 0x02   /* a listed KV block lies outside [0, ceil(seqused_kv/128)); skipped */
#define GBSA_DEV_BAD_COUNT 0x04       /* sparse_count outside [0, top_k]; clamped                       */
#define GBSA_DEV_BAD_PAGE 0x08        /* block_table entry outside [0, num_pages); the page reads as 0  */
#define GBSA_DEV_META_MISMATCH 0x10   /* metadata built for another problem; forward did nothing         */
#define GBSA_DEV_TIMEOUT 0x20         /* a pipeline wait gave up (wait_limit_ns); results are not valid   */
#define GBSA_DEV_CAPACITY 0x40        /* a work-list capacity bound was exceeded; forward did nothing    */

/* Host-known description of one call.  No field is read from the device.
 * Field names follow the GBSA article's aclnn and PyTorch signatures
 * ("Calling / aclnn API", "Calling / PyTorch API"). */
typedef struct gbsa_problem {
  int32_t B;                  /* number of sequences (batch)                                  */
  int32_t T;                  /* total query tokens = cu_seqlens_q[B]                         */
  int32_t N1;                 /* query heads                                                  */
  int32_t N2;                 /* key/value heads; N1 % N2 == 0, N1/N2 <= 128                  */
  int32_t D;                  /* head dim; only 128 ("Constraints: dimension")                */
  int32_t block_x;            /* blockShapeX: query tokens per Q block, >= 1                  */
  int32_t block_y;            /* blockShapeY: keys per KV block; must equal the page size 128 */
  int32_t total_q_blocks;     /* sum_b ceil(storage_len_b / block_x)                          */
  int32_t top_k;              /* last dim of sparse_idx; 1..256                               */
  int32_t max_pages_per_seq;  /* second dim of block_table                                    */
  int32_t num_pages;          /* first dim of the K/V pool                                    */
  int64_t kv_page_stride;     /* elements between pages; >= 128*N2*D and % (N2*D) == 0        */
  double scale;               /* scale_value; 0.0 selects 1/sqrt(D)                           */
  int32_t mask_mode;          /* 1 = built-in causal (the only mode the article supports)    */
  int32_t win_left;           /* -1 = unbounded; else keys >= pos - win_left are kept         */
  int32_t win_right;          /* -1 = unbounded; else keys <= pos + win_right are kept        */
  int32_t is_packed_gqa;      /* 1: the G heads of a group share each K/V tile; 0 (a head per
                                 tile) is accepted and gives the same rows: the library always
                                 packs, and no row's arithmetic depends on the packing        */
  int32_t return_lse;         /* 1: write lse                                                 */
  int32_t has_seqused_q;      /* 1: seqused_q is given; 0: every Q storage token is used      */
  int32_t num_ctas;           /* persistent CTAs of the forward; 0 = SM count of the device   */
  int32_t max_blocks_per_split; /* 0 = automatic split-KV length; > 0 forces a smaller one     */
  int32_t dtype;              /* element type of q, k, v: GBSA_DTYPE_BF16, _FP16, _FP8_E4M3   */
  int32_t softmax_precision;  /* softmaxPrecision: 0 = fp32 online softmax; 1 (the article's
                                 half-precision softmax with fp32 rescale) is accepted and
                                 computed with the fp32 softmax, whose error is smaller   */
  int32_t kv_layout;          /* GBSA_KV_PAGED (k, v: the page pool, block_table) or
                                 GBSA_KV_TND (k, v: [T_kv, N2, D], cu_seqlens_kv)             */
  int32_t T_kv;               /* GBSA_KV_TND: rows of k and v (= cu_seqlens_kv[B]); else 0   */
  double q_scale;             /* GBSA_DTYPE_FP8_E4M3: per-tensor dequantization scales, each */
  double k_scale;             /*   finite and > 0 (q = q_scale * code, ...); the other dtypes */
  double v_scale;             /*   ignore them                                                 */
  int64_t wait_limit_ns;      /* bound of every pipeline wait of the forward kernel, in ns;
                                 0 = 1 s.  A wait that runs out sets GBSA_DEV_TIMEOUT, and the
                                 kernel drains the copies and MMAs it issued and returns
                                 (results invalid).  The clock starts after the wait's first
                                 barrier probe, which the hardware may hold for tens of us:
                                 a wait gives up no earlier than the bound.  >= 0; ABI 5      */
} gbsa_problem;

/* K/V layouts (GBSA article, "Constraints: layouts": PA_BBND page pool, or
 * TND with cuSeqLengthsKv).  TND: sequence b's keys are rows
 * [cu_seqlens_kv[b], cu_seqlens_kv[b+1]) of k and v, contiguous, and a
 * "block" lb of its list is rows cu_seqlens_kv[b] + 128*lb ...; block_table,
 * num_pages, max_pages_per_seq and kv_page_stride are unused.  seqused_kv is
 * required in both layouts and must not exceed the sequence's TND rows. */
#define GBSA_KV_PAGED 0
#define GBSA_KV_TND 1

/* Element types (GBSA article, "Constraints: data types": bf16 and fp16 for
 * Q, K, V and the output; lse is fp32 either way).  Accumulation is fp32.
 * GBSA_DTYPE_FP8_E4M3 (the article's quantised-input arguments, with one
 * dequantization scale per tensor): q, k, v hold E4M3 codes (1 byte, no
 * infinity, S.1111.111 = NaN), scores are (q_scale*q).(k_scale*k)*scale, the
 * softmax weights are rounded to E4M3 (times 2^8) for the P.V product, and
 * out is bf16 holding softmax(.) (v_scale*v).  Expected error per element:
 * about 2^-4 of sum_p w_p |v_scale*v_p| (the weights' E4M3 rounding). */
#define GBSA_DTYPE_BF16 0
#define GBSA_DTYPE_FP16 1
#define GBSA_DTYPE_FP8_E4M3 2

/* Device pointers of one call (caller-owned).  Unused optional pointers are NULL. */
typedef struct gbsa_tensors {
  const void* q;               /* dtype [T, N1, D] (E4M3: 1 byte per element)     */
  const void* k;               /* dtype [num_pages, 128, N2, D], page stride above*/
  const void* v;               /* same layout and stride as k                     */
  const int32_t* sparse_idx;   /* [N2, total_q_blocks, top_k]                     */
  const int32_t* sparse_count; /* [N2, total_q_blocks]                            */
  const int64_t* cu_seqlens_q; /* [B+1]                                           */
  const int32_t* seqused_q;    /* [B] or NULL (has_seqused_q = 0)                 */
  const int32_t* seqused_kv;   /* [B]                                             */
  const int32_t* block_table;  /* [B, max_pages_per_seq]                          */
  void* out;                   /* [T, N1, D]: fp16 for FP16, else bf16            */
  float* lse;                  /* fp32 [T, N1] or NULL (return_lse = 0)           */
  const int64_t* cu_seqlens_kv; /* [B+1] for GBSA_KV_TND, else NULL               */
} gbsa_tensors;

/* Version of this header the library was built from (GBSA_ABI_VERSION). */
GBSA_API int32_t gbsa_abi_version(void);

/* Human-readable name of a status code; never NULL. */
GBSA_API const char* gbsa_status_string(gbsa_status status);

/* Bytes of metadata gbsa_metadata() writes for `problem` (a host-known bound:
 * it does not depend on device values).  Validates `problem` first.
 * GBSA article, "two-phase call": the metadata records the core split.
 * Returns GBSA_ERR_NO_DEVICE if num_ctas == 0 and no device can be queried. */
GBSA_API gbsa_status gbsa_metadata_size(const gbsa_problem* problem, size_t* bytes);

/* Up to this many sequences (B) gbsa_metadata() launches two kernels on the
 * stream (items with their own sequence phase, then the plan); above it,
 * three (a sequence kernel first).  The bytes written are the same. */
#define GBSA_METADATA_FUSED_MAX_B 1024

/* Builds the work list for `problem` into the caller's device buffer `meta`
 * (16-byte aligned, meta_bytes >= gbsa_metadata_size()).  Reads
 * sparse_idx, sparse_count, cu_seqlens_q, seqused_q and seqused_kv; other
 * tensor fields may be NULL.  Deterministic: equal inputs give equal bytes.
 * The buffer's previous content is irrelevant (nothing has to be zeroed).
 * GBSA article, "two-phase call" step 2 and "Constraints: metadata first". */
GBSA_API gbsa_status gbsa_metadata(const gbsa_problem* problem, const gbsa_tensors* tensors,
                          void* meta, size_t meta_bytes, int32_t* dev_status, void* stream);

/* Bytes of scratch the forward needs for split-KV partial results
 * (fp32 partial outputs and log-sum-exps); may be 0 only if splitting is
 * impossible.  GBSA article, "aclnn API": first-phase workspace query. */
GBSA_API gbsa_status gbsa_workspace_size(const gbsa_problem* problem, size_t* bytes);

/* Runs the attention: out (and lse when return_lse) from q, k, v through the
 * work list in `meta`.  `workspace` (16-byte aligned, ws_bytes >=
 * gbsa_workspace_size()) is caller-owned scratch, overwritten.  If `meta`
 * was built for a different problem the kernels set GBSA_DEV_META_MISMATCH
 * and leave out/lse (and `meta`) untouched.
 * The forward writes to `meta` (ABI 6): the CTAs take work units through a
 * counter in its header (words 26 and 27), which gbsa_metadata() leaves at
 * zero and every forward call puts back to zero before it finishes, so the
 * same metadata serves any number of calls, CUDA graph replays included.
 * Calls that share one metadata buffer must therefore not overlap on the GPU
 * (other streams, other host threads): order them on one stream or with
 * events, or give each its own copy.  Deterministic for a fixed num_ctas
 * (GBSA article, "Constraints: determinism").  Rows past seqused_q, and rows
 * with no visible key, get out = 0 and lse = -inf. */
GBSA_API gbsa_status gbsa_forward(const gbsa_problem* problem, const gbsa_tensors* tensors,
                         void* meta, void* workspace, size_t ws_bytes,
                         int32_t* dev_status, void* stream);

/* Size of the device scratch that gbsa_forward_static_scratch() uses. */
#define GBSA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* gbsa_forward() for callers that cannot allocate device memory (the paper
 * has no counterpart: this is a library addition).  Some hosts hand out a
 * fixed device-memory budget at start-up and forbid any allocation later,
 * and code that runs inside an allocator or a framework hook cannot call
 * cudaMalloc without risking a deadlock; such callers have no way to provide
 * the workspace gbsa_forward() asks for.  Here the split-KV scratch is a
 * GBSA_STATIC_SCRATCH_BYTES array that the library's CUDA module holds on
 * every GPU that loads it, until the process exits; nothing is allocated,
 * and the caller still passes inputs, outputs and the metadata.
 *   - Limit: problems whose gbsa_workspace_size() exceeds
 *     GBSA_STATIC_SCRATCH_BYTES are rejected with GBSA_ERR_WORKSPACE_TOO_SMALL
 *     before anything is launched (decode-shaped problems fit; prefill-shaped
 *     ones need gbsa_forward() with a caller-provided workspace).
 *   - The array comes into being when the CUDA module holding it is loaded
 *     in a context.  With lazy module loading (the CUDA default) that is the
 *     first call of this entry point on a device: that call loads the module,
 *     which reserves GBSA_STATIC_SCRATCH_BYTES of device memory, and looks up
 *     the array's device address.  A caller with a fixed memory budget should
 *     make one call during start-up, before the budget is fixed, and make
 *     that first call before any stream capture on that device.  The address
 *     is looked up again when another context of the device is current (for
 *     instance after cudaDeviceReset), which loads the module there too.
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents (nothing in it needs to start at zero: every partial the
 *     merge reads is written earlier in the same call).  Calls whose work
 *     overlaps on the GPU (other streams, other host threads) race on it:
 *     order them on one stream or with events.
 * Everything else -- arguments, layouts, errors, dev_status -- is as for
 * gbsa_forward(). */
GBSA_API gbsa_status gbsa_forward_static_scratch(const gbsa_problem* problem,
                                                 const gbsa_tensors* tensors, void* meta,
                                                 int32_t* dev_status, void* stream);

/* Bytes of device scratch gbsa_backward() needs: one fp32 per (token, query
 * head), T * N1 * 4 rounded up to 16. */
GBSA_API gbsa_status gbsa_backward_workspace_size(const gbsa_problem* problem, size_t* bytes);

/* Gradients of the attention output, for training (the GBSA article's
 * overview names training as a use of the operator but specifies no
 * backward; this is the exact gradient of the forward's function, a
 * library addition).  Given dout (the gradient of the loss with respect to
 * out: [T][N1][D], the element type of q) it computes
 *   dq [T][N1][D]                       fp32, every row written (0 where a
 *                                       row has no visible key or lies past
 *                                       seqused_q);
 *   dk, dv                              fp32, compact: [num_pages][128][N2][D]
 *                                       for the paged pool (page p's rows at
 *                                       p * 128 * N2 * D, whatever the pool's
 *                                       kv_page_stride), or [T_kv][N2][D] for
 *                                       TND; zeroed by the call, then summed
 *                                       over every row and list entry that
 *                                       reads a key (a block listed twice
 *                                       counts twice, as in the forward).
 * Inputs are those of the forward call plus its results: tensors->out and
 * tensors->lse (lse required, whatever problem->return_lse says) for the
 * same q, k, v and lists; `meta` is the work list gbsa_metadata() built for
 * this problem (read only here).  bf16 and fp16 only (E4M3:
 * GBSA_ERR_UNSUPPORTED); softmax_precision is ignored (the gradient of the
 * exact softmax).  `workspace` (16-byte aligned, ws_bytes >=
 * gbsa_backward_workspace_size()) is overwritten.  All pointers 16-byte
 * aligned except lse (4).  Errors as for gbsa_forward(); a page index out of
 * range sets GBSA_DEV_BAD_PAGE and skips the block. */
GBSA_API gbsa_status gbsa_backward(const gbsa_problem* problem, const gbsa_tensors* tensors,
                                   const void* dout, const void* meta, float* dq, float* dk,
                                   float* dv, void* workspace, size_t ws_bytes,
                                   int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GBSA_H */
