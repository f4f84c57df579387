/*
 * libq4dec -- Q4_0 decode hot path for NVIDIA B200 (sm_100a).
 *
 * Two operations make up one decode step of a quantised dense model:
 *
 *  1. q4_gemv: a dequant-fused GEMV / skinny GEMM that streams Q4_0 weights
 *     once for M = 1..5 activation rows.  The pages ("Qwen3.8-27B at 256K on
 *     a 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", the paragraph
 *     beginning "NVIDIA quotes 432 GB/s") put decode time into "repeatedly
 *     streaming quantized weights"; M = 1 is plain decode and M = 2..5 is the
 *     target model verifying a drafted block of up to four tokens
 *     ("Qwen3.8-27B on RTX 4090: 5,000 tok/s Prefill Reproduced", section
 *     "MTP helps ordinary prose, but acceptance controls the gain").
 *
 *  2. q4kv_attn_decode: causal GQA flash-decode attention over a K/V cache
 *     stored in the same Q4_0 layout (same first page: "With Q4 K and V ..."
 *     and "the 16 attention layers add increasingly expensive KV reads as
 *     context fills").  The context is split across the SMs and the partial
 *     softmax states are combined by a log-sum-exp merge.
 *
 * Around them: q4_gemv_swiglu_ex (the feed-forward block's gate and up
 * projections in one weight stream, with the SwiGLU epilogue), q4kv_append
 * (quantises the verified tokens' K/V rows into the cache), and
 * q8kv_attn_decode_ex (the same attention over an 8-bit Q8_0 cache).
 *
 * ---------------------------------------------------------------------------
 * Storage layout (identical for weights and for the K/V cache)
 *
 *   Q4_0 block   : 32 elements, one IEEE fp16 scale d, 16 bytes of nibbles.
 *                  Byte j (0..15) holds element j in bits 0..3 and element
 *                  j+16 in bits 4..7.  Element value = d * (q - 8), q in 0..15.
 *   super-block  : 256 consecutive elements = 8 blocks in 144 bytes:
 *                  bytes [16*b, 16*b+16) = nibbles of block b (b = 0..7),
 *                  bytes [128+2*b, 128+2*b+2) = fp16 scale of block b
 *                  (little endian).  144 is a multiple of 16, so every
 *                  super-block starts on a 16-byte boundary.
 *   weight W[N][K]: super-block-column-major: K/256 columns one after
 *                  another, column s holding super-block s of rows 0..N-1,
 *                  so super-block (n, s) starts at byte (s*N + n) * 144.
 *                  (The rows a GPU block streams are then contiguous in
 *                  every column.)  A row-major Q4_0 matrix converts by
 *                  moving whole 144-byte super-blocks.
 *   K/V cache    : one super-block per (KV head, token) (head_dim = 256);
 *                  token t of KV head h starts at byte (h*kv_stride + t)*144.
 *
 * Conventions
 *   - Every pointer passed to a compute entry point is a DEVICE pointer of
 *     the current CUDA device, owned by the caller; the library never frees
 *     or retains it.  W, x, Q, K, V and workspace must be 16-byte aligned;
 *     y and out must be 4-byte aligned (2-byte for bf16 outputs).
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; the library never
 *     synchronises the host on the compute path.
 *   - Arguments are validated before anything is launched; on any error
 *     nothing is launched and the outputs are untouched.  Launch failures
 *     return Q4D_ERR_CUDA.  Faults during execution surface at the caller's
 *     next synchronisation.  Every wait inside a kernel is bounded in time;
 *     a wait that runs out sets a device error word readable through
 *     q4d_device_error().
 *   - Results are fp32 (the GEMVs store bf16 on request).  Accumulation is
 *     fp32; the kernels use no atomics on results, so repeated calls with
 *     the same inputs and the same device give bitwise identical outputs.
 */
#ifndef Q4DEC_H
#define Q4DEC_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define Q4D_VERSION 20000 /* 2.0.0 */

typedef enum {
  Q4D_OK = 0,
  Q4D_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad scale */
  Q4D_ERR_UNSUPPORTED_SHAPE = 2, /* M outside 1..5, K % 256 != 0, head_dim != 256,
                                    n_q % n_kv != 0, ctx_len < M, stride < ctx_len */
  Q4D_ERR_MISALIGNED = 3,        /* pointer alignment below the stated minimum */
  Q4D_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required */
  Q4D_ERR_CUDA = 5,              /* CUDA runtime error (launch, device query, malloc) */
  Q4D_ERR_DEVICE_TIMEOUT = 6,    /* a bounded in-kernel wait ran out (q4d_device_error) */
  Q4D_ERR_DEVICE_INDEX = 7       /* an index check of a debug build failed (q4d_device_error) */
} q4d_status;

/* Library version, Q4D_VERSION of the build. */
int q4d_version(void);

/* Static, never-NULL description of a status code (unknown codes included). */
const char* q4d_status_string(int status);

/* ------------------------------------------------------------------ GEMV --
 * y[m][n] = sum_k (d * (q - 8))[n][k] * x[m][k]   for m < M, n < N.
 *
 *   W_q4 : N x K elements of Q4_0 in the weight layout above, N*K/256*144 bytes.
 *   x    : bf16 [M][K] row-major (M activation rows sharing one weight stream).
 *   y    : fp32 [M][N] row-major, fully overwritten.
 *   Requirements: 1 <= M <= 5, N >= 1, K >= 256, K % 256 == 0.
 *
 * q4_gemv runs on the legacy default stream with a workspace owned by the
 * library (per device, allocated on first need and grown when a larger one
 * is needed -- that call synchronises the device and must not be captured
 * into a CUDA graph).  q4_gemv_ex takes the stream and a caller-owned
 * workspace of at least q4d_gemv_workspace_bytes(M, N, K) bytes (it may be
 * NULL when that size is 0); it never allocates.
 *
 * Partition (q4d_plan_gemv): rows are cut into blocks of 128 and K into units
 * of 512 elements; the units are shared out in equal contiguous ranges over
 * one CTA per SM, so a row block may be summed by several CTAs.  All but
 * one of them write their fp32 partial sums into the workspace, each entry
 * (8 bytes) holding a partial sum and the launch's tag, which marks it as
 * written; the CTA whose range ends in the row block waits until the entries
 * carry the tag, adds the partial sums in a fixed (K) order, so results are
 * deterministic, and clears the entries.  The workspace must therefore be zero-filled before
 * its first use; every launch that returns Q4D_OK and leaves the device error
 * word at 0 leaves it zero-filled again, so one zeroing serves any number of
 * GEMV calls of any shape (zero it again after a reported error, and do not
 * share it with other kernels).  Calls whose kernels may overlap on the GPU
 * must not share one workspace.  The library's own workspace (q4_gemv) is
 * zeroed when allocated.
 */
q4d_status q4_gemv(const void* W_q4, const void* x, float* y, int M, int N, int K);
q4d_status q4_gemv_ex(const void* W_q4, const void* x, float* y, int M, int N, int K,
                      void* stream, void* workspace, size_t workspace_bytes);

/* q4_gemv_ex2: q4_gemv_ex plus flags (0 behaves exactly as q4_gemv_ex; a bit
 * other than the two below is Q4D_ERR_INVALID_ARG).
 *
 *   Q4D_GEMV_WEIGHT_PREFETCH: launch with programmatic dependent launch.  The
 *   kernel's CTAs may start while the kernel before it on the stream is still
 *   running, and stream the first pipeline stages of W_q4 at once; they read
 *   x, and write y and the workspace, only after that kernel has completed
 *   and its writes are visible.  The caller guarantees that no kernel issued
 *   earlier on the stream still writes W_q4 (true for inference weights).
 *   Back-to-back GEMVs then overlap one call's start-up with the previous
 *   call's tail.  No counterpart in the source pages: a launch-time option of
 *   this library.
 */
#define Q4D_GEMV_WEIGHT_PREFETCH 1u
/*   Q4D_GEMV_OUT_BF16: y is bf16 [M][N] (2 bytes per element, 2-byte
 *   aligned) instead of fp32: each element is the fp32 result of the plain
 *   call rounded to nearest even -- bit for bit the fp32 output converted --
 *   so that a GEMV's output can feed the next GEMV's bf16 activations
 *   directly.  A K split still reduces its partials in fp32 (the workspace
 *   size does not change).  No counterpart in the source pages, which keep
 *   activations in 16 bits between layers without fixing the format.
 */
#define Q4D_GEMV_OUT_BF16 2u
q4d_status q4_gemv_ex2(const void* W_q4, const void* x, void* y, int M, int N, int K,
                       void* stream, void* workspace, size_t workspace_bytes, unsigned flags);

/* q4_gemv_swiglu_ex: fused gate / up projections with the SwiGLU epilogue of
 * a gated feed-forward block ("Qwen3.8-27B at 256K on a 24GB RTX PRO 4000 SFF
 * (432 GB/s): 50 tok/s with MTP": the FFN's gate, up and down projections).
 *
 *   W_gu : 2N x K elements of Q4_0 in the weight layout above, the gate row n
 *          stored as row 2n and the up row n as row 2n + 1 (interleaved).
 *   x    : bf16 [M][K];  h : fp32 [M][N] = silu(g) * u, silu(g) = g / (1 + e^-g)
 *          evaluated in fp32 with expf, g and u the fp32 gate / up outputs of
 *          row pair n (bf16 [M][N] with Q4D_GEMV_OUT_BF16: the fp32 h rounded
 *          to nearest even).
 *   Requirements as q4_gemv (with 2N rows); workspace of at least
 *   q4d_gemv_swiglu_workspace_bytes(M, N, K) bytes; flags as q4_gemv_ex2.
 * One weight stream and one launch instead of two GEMVs and an elementwise
 * pass.
 */
q4d_status q4_gemv_swiglu_ex(const void* W_gu, const void* x, void* h, int M, int N, int K,
                             void* stream, void* workspace, size_t workspace_bytes,
                             unsigned flags);
size_t q4d_gemv_swiglu_workspace_bytes(int M, int N, int K);
/* Workspace bytes q4_gemv_ex needs on the CURRENT device (depends on its SM
 * count; a host without a usable device is planned for 148 SMs).  Returns 0
 * for invalid shapes as well as for shapes that need none. */
size_t q4d_gemv_workspace_bytes(int M, int N, int K);

/* ------------------------------------------------------------ GEMV batch --
 * Many GEMVs in ONE launch: the weight stream of a whole decode step (every
 * layer's projections and the output head, "Qwen3.8-27B at 256K on a 24GB RTX
 * PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraph beginning "NVIDIA
 * quotes 432 GB/s") without a launch, ramp-up and tail per matrix.  The jobs
 * run in order on one CTA per SM; while a job waits for its input, the CTAs
 * already stream the weights of the jobs after it (weights depend on
 * nothing).  No counterpart in the pages: a launch form of this library.
 *
 *   q4d_gemv_job: one GEMV of the batch.
 *     W_q4, x, y, N, K : as q4_gemv (device pointers; y is [M][N]);
 *     flags   : Q4D_GEMV_OUT_BF16 (y in bf16) and/or Q4D_GEMV_SWIGLU (W_q4
 *               holds 2N interleaved gate / up rows and y receives
 *               h = silu(g) * u [M][N], as q4_gemv_swiglu_ex);
 *     wait_for: -1 -- x may be read as soon as the kernel before the launch on
 *               the stream has completed (every job can use -1 when no job of
 *               the batch writes another job's x);
 *               j (0 <= j < this job's index) -- x is read only after job j
 *               has written all of its output, e.g. x is job j's y.  Only job
 *               j is waited for: a job that reads the outputs of several
 *               earlier jobs needs them ordered by a chain of waits (job j
 *               itself waiting, directly or through others, for the rest).
 *   Each job must also not overwrite an x or y that an earlier job, not yet
 *   finished, still uses: make it wait, directly or through a chain of
 *   waits, for that job.
 *
 *   q4d_gemv_batch_desc_bytes(n_jobs): bytes of the launch descriptor.
 *   q4d_gemv_batch_prepare: host only (no CUDA call).  Validates every job as
 *     q4_gemv would (same status codes), plans the launch for a device with
 *     num_sms SMs and M activation rows (every job has M rows), writes the
 *     descriptor into the host buffer `desc` (desc_bytes >= the size above)
 *     and the workspace size into *workspace_bytes.
 *   q4_gemv_batch_ex: launches the batch on `stream`.  desc_host is the
 *     prepared host buffer, desc_dev a byte-for-byte copy of it in device
 *     memory (16-byte aligned): copy it once, launch many times.  Its tail
 *     holds the per-job completion counters (row-block halves written in
 *     final form), zero as prepared; a launch counts on them and sets them
 *     back to zero before it ends, so launches that may overlap on the GPU
 *     must not share a descriptor copy, and a copy must not be rewritten while
 *     a launch may run.  num_sms
 *     must be the current device's SM count, else Q4D_ERR_INVALID_ARG.
 *     workspace: device memory of at least *workspace_bytes (16-byte aligned;
 *     zero-filled before first use and kept so, as for q4_gemv_ex; launches
 *     that may overlap on the GPU must not share it), else
 *     Q4D_ERR_WORKSPACE.  flags: 0 or
 *     Q4D_GEMV_WEIGHT_PREFETCH (as q4_gemv_ex2: the first weights stream while
 *     the previous kernel on the stream still runs).  Never allocates; the
 *     launch can be captured into a CUDA graph and replayed.
 *   The CTAs of a batch wait for one another between dependent jobs, so all
 *   of them must be resident together: one CTA per SM, as launched, on an
 *   otherwise idle device (each wait is bounded; see q4d_device_error).
 *   Results are those of the single-GEMV entry points, bit for bit.
 */
#define Q4D_GEMV_SWIGLU 4u
typedef struct {
  const void* W_q4;
  const void* x;
  void* y;
  int N;
  int K;
  unsigned flags;
  int wait_for;
} q4d_gemv_job;
size_t q4d_gemv_batch_desc_bytes(int n_jobs);
q4d_status q4d_gemv_batch_prepare(const q4d_gemv_job* jobs, int n_jobs, int M, int num_sms,
                                  void* desc, size_t desc_bytes, size_t* workspace_bytes);
q4d_status q4_gemv_batch_ex(const void* desc_host, void* desc_dev, void* stream,
                            void* workspace, size_t workspace_bytes, unsigned flags);

/* ------------------------------------------------------------- attention --
 * For draft row m (absolute position p_m = ctx_len - M + m) and query head h
 * (KV head kh = h / (n_q_heads / n_kv_heads)):
 *   s[t]        = softmax_scale * sum_c Q[m][h][c] * Khat[kh][t][c],  t <= p_m
 *   out[m][h][:] = sum_t softmax(s)[t] * Vhat[kh][t][:]
 * where Khat / Vhat are the dequantised caches.  Tokens t > p_m are masked
 * (the M draft tokens are already in the cache; row M-1 sees all ctx_len).
 *
 *   Q    : bf16 [M][n_q_heads][head_dim].
 *   Kq4, Vq4 : [n_kv_heads][kv_stride] super-blocks (one per token, 144 B).
 *   out  : fp32 [M][n_q_heads][head_dim], fully overwritten.
 *   Requirements: head_dim == 256, 1 <= M <= 5, n_kv_heads >= 1,
 *                 n_q_heads % n_kv_heads == 0, ctx_len >= M,
 *                 kv_stride_tokens >= ctx_len, softmax_scale finite.
 *
 * q4kv_attn_decode uses kv_stride = ctx_len, softmax_scale = 1 (queries are
 * pre-scaled), the legacy default stream and a library-owned workspace (same
 * rules as q4_gemv).  The _ex form takes all of them explicitly and never
 * allocates; workspace must hold q4d_attn_workspace_bytes(...) bytes.
 *
 * Supported value range (the same for every M and both cache formats): the
 * kernels feed Q and the dequantised K/V values to the tensor cores as IEEE
 * fp16, so
 *   - |Q| <= 65504 (bf16 queries beyond the fp16 range are not supported;
 *     |Q| < 2^-14 is rounded to an fp16 subnormal, absolute error <= 2^-25);
 *   - Q4_0 cache: |d| <= 8188 for every block scale, so that every value
 *     d * (q - 8) lies within +-65504 (q4kv_append stores such scales for
 *     any input |v| <= 65504);
 *   - Q8_0 cache: |d| <= 511.75, so that every value d * q (q = -128..127)
 *     lies within +-65504.
 * Inside this range the result meets the stated accuracy for any row count;
 * outside it the result is undefined (it may be inf or NaN).  The scales are
 * device data, so the library does not check them.
 */
q4d_status q4kv_attn_decode(const void* Q, const void* Kq4, const void* Vq4, float* out,
                            int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M);
q4d_status q4kv_attn_decode_ex(const void* Q, const void* Kq4, const void* Vq4, float* out,
                               int ctx_len, int n_q_heads, int n_kv_heads, int head_dim,
                               int M, int kv_stride_tokens, float softmax_scale,
                               void* stream, void* workspace, size_t workspace_bytes);
/* Workspace bytes q4kv_attn_decode_ex needs on the current device (0 for
 * invalid shapes and for shapes handled in one pass). */
size_t q4d_attn_workspace_bytes(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim,
                                int M);

/* -------------------------------------------- attention, Q8_0 K/V cache --
 * The same attention over the 8-bit cache type the page "Running
 * Qwen3.8-27B on an RTX 4090" launches its server with (--cache-type-k /
 * --cache-type-v q8_0): Q8_0 blocks of 32 int8 values q and one fp16 scale d,
 * value d * q.
 *
 *   Kq8, Vq8 : [n_kv_heads][kv_stride_tokens] 272-byte super-blocks, one per
 *              token: bytes 0..255 the int8 values (element j of block b at
 *              byte 32*b + j, two's complement), bytes 256 + 2*b the fp16
 *              scale of block b (little endian); 16-byte aligned.
 *   Everything else (Q, out, requirements, workspace, errors) as
 *   q4kv_attn_decode_ex, with the workspace size from
 *   q8kv_attn_workspace_bytes.  Every row count runs on the tensor-memory
 *   kernel; K and V enter the tensor core as fp16 d * q, each rounded once.
 */
q4d_status q8kv_attn_decode_ex(const void* Q, const void* Kq8, const void* Vq8, float* out,
                               int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                               int kv_stride_tokens, float softmax_scale, void* stream,
                               void* workspace, size_t workspace_bytes);
size_t q8kv_attn_workspace_bytes(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim,
                                 int M);

/* ------------------------------------------- attention, allocation-free --
 * The pages have no counterpart to this entry point; it exists for deployment.
 *
 * Some callers may not allocate device memory once they are running: runtimes
 * that reserve all device memory in their own arena at start-up and forbid
 * allocation afterwards, and latency-critical decode loops in which a
 * cudaMalloc/cudaFree would synchronise the device and stall the token.  They
 * cannot use q4kv_attn_decode (which may allocate its workspace) and may have
 * no spare buffer to hand to the _ex form.  This entry point takes no
 * workspace and allocates nothing: the per-split softmax states live in one
 * statically sized device array of Q4D_NOALLOC_SCRATCH_BYTES inside this
 * library, which every GPU that loads the library holds until the process
 * exits.
 *
 *   - Arguments, layout and results are those of q4kv_attn_decode_ex without
 *     the workspace.  A call needing more scratch than the array holds
 *     (q4d_attn_workspace_bytes > Q4D_NOALLOC_SCRATCH_BYTES) returns
 *     Q4D_ERR_WORKSPACE and launches nothing.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (each call writes every state it
 *     reads), but calls whose kernels overlap on the GPU -- e.g. on two
 *     streams without ordering between them -- race and give wrong results.
 */
#define Q4D_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB */
q4d_status q4kv_attn_decode_noalloc(const void* Q, const void* Kq4, const void* Vq4, float* out,
                                    int ctx_len, int n_q_heads, int n_kv_heads, int head_dim,
                                    int M, int kv_stride_tokens, float softmax_scale,
                                    void* stream);

/* ------------------------------------------------------- launch planning --
 * Pure host functions (no CUDA call) exposing how a call is partitioned on
 * a device with num_sms SMs; the compute entry points use exactly these.
 */
typedef struct {
  int grid;              /* CTAs, one per SM at most (fewer only for tiny shapes)  */
  int threads;           /* threads per CTA                                        */
  int row_blocks;        /* ceil(N / 128): blocks of 128 weight rows               */
  int units_per_row_block; /* ceil(K / 512): units of two 256-element columns      */
  int units;             /* row_blocks * units_per_row_block, shared out evenly    */
  int slots;             /* most CTAs sharing one row block (0: none is shared)    */
  int stages;            /* shared-memory pipeline depth (one unit per stage)      */
  int reserved;
  size_t smem_bytes;     /* dynamic shared memory per CTA                          */
  size_t workspace_bytes;/* tagged 8-byte partial-sum entries of shared row blocks */
} q4d_gemv_plan;

typedef struct {
  int n_splits;          /* context splits per KV head                           */
  int split_tokens;      /* tokens per split (multiple of tile_tokens)           */
  int tile_tokens;       /* tokens per shared-memory tile                        */
  int row_groups;        /* CTAs per (KV head, split) when g*M exceeds one CTA   */
  int rows_per_cta;      /* query rows (draft rows x grouped heads) per CTA      */
  int stages;            /* shared-memory pipeline depth                         */
  int threads;           /* threads per CTA                                      */
  size_t smem_bytes;     /* dynamic shared memory per CTA                        */
  size_t workspace_bytes;/* partial (max, sum, o[256]) states for the merge      */
} q4d_attn_plan;

q4d_status q4d_plan_gemv(int M, int N, int K, int num_sms, q4d_gemv_plan* plan);
q4d_status q4d_plan_attn(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                         int num_sms, q4d_attn_plan* plan);
/* The plan of q8kv_attn_decode_ex (the Q8_0 cache). */
q4d_status q8kv_plan_attn(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                          int num_sms, q4d_attn_plan* plan);

/* ------------------------------------------------------- K/V append --
 * Quantise the K and V rows of M new tokens and write them at token positions
 * pos .. pos+M-1 of every KV head of the Q4_0 caches ("Qwen3.8-27B at 256K on
 * a 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraph on the
 * 16 full-attention layers: the K/V cache is Q4 and grows by the verified
 * tokens).  Per 32-element block: amax = the element of largest magnitude
 * (first on ties), d = fp16(amax / -8), q = clamp(floor(v/d + 8.5), 0, 15)
 * with the division and addition rounded to nearest in fp32; a zero d is
 * stored as +0 with every q = 8.
 *
 *   Kq4, Vq4     : caches, [n_kv_heads][kv_stride_tokens] super-blocks (head_dim 256).
 *   k_new, v_new : fp32 [M][n_kv_heads][256], device pointers.
 *   Requirements: n_kv_heads >= 1, M >= 1, pos >= 0, pos + M <= kv_stride_tokens;
 *   caches 16-byte and k_new / v_new 4-byte aligned.  Runs on `stream`
 *   (NULL = legacy default stream); allocates nothing; only the M target
 *   tokens' super-blocks are written.
 *   Errors: Q4D_ERR_INVALID_ARG, Q4D_ERR_UNSUPPORTED_SHAPE (pos + M beyond
 *   the stride), Q4D_ERR_MISALIGNED, Q4D_ERR_CUDA; nothing is launched on error.
 */
q4d_status q4kv_append(void* Kq4, void* Vq4, const float* k_new, const float* v_new,
                       int n_kv_heads, int kv_stride_tokens, int pos, int M, void* stream);

/* ------------------------------------------------ host layout helpers --
 * Conversions between the canonical 18-byte Q4_0 block (GGUF order: fp16 d,
 * little endian, then 16 bytes where byte j holds element j in its low nibble
 * and element j + 16 in its high nibble) and this library's 144-byte
 * super-block (the 8 blocks' 16 nibble bytes, then their 8 fp16 scales).
 * The canonical input is row-major: rows of K/32 blocks.  Plain host code on
 * host pointers, no CUDA; no counterpart on the source pages (format
 * plumbing for data quantised elsewhere).
 *
 *   q4d_pack_q4_0_weights:   blocks18 [N][K/32] -> W_q4 in the weight layout
 *                            (super-block (n, s) at byte (s*N + n) * 144).
 *   q4d_unpack_q4_0_weights: the inverse.
 *   q4d_pack_q4_0_rows:      blocks18 [rows][K/32] -> rows of super-blocks in
 *                            row order (super-block (r, s) at (r*K/256 + s) * 144),
 *                            the K/V cache layout (one row per token, K = 256).
 *   q4d_unpack_q4_0_rows:    the inverse.
 * Requirements: non-null pointers, rows (N) >= 1, K >= 256, K % 256 == 0; the
 * buffers hold rows*K/32*18 and rows*K/256*144 bytes and do not overlap.
 * Errors: Q4D_ERR_INVALID_ARG (null, rows < 1), Q4D_ERR_UNSUPPORTED_SHAPE (K).
 */
q4d_status q4d_pack_q4_0_weights(const void* blocks18, void* W_q4, int N, int K);
q4d_status q4d_unpack_q4_0_weights(const void* W_q4, void* blocks18, int N, int K);
q4d_status q4d_pack_q4_0_rows(const void* blocks18, void* rows_q4, int rows, int K);
q4d_status q4d_unpack_q4_0_rows(const void* rows_q4, void* blocks18, int rows, int K);

/* ------------------------------------------------------- device errors --
 * Synchronises the current device and reads the library's device error
 * record: a word of bits (1: an in-kernel wait exceeded its time limit; 2: an
 * index check of a debug build failed) and the first failed index check.
 * Returns Q4D_OK when clear, Q4D_ERR_DEVICE_INDEX when bit 2 is set, else
 * Q4D_ERR_DEVICE_TIMEOUT when bit 1 is set, Q4D_ERR_CUDA if the device
 * cannot be queried.  reset != 0 clears the record after reading.
 */
q4d_status q4d_device_error(int reset);

/* The same, also copying the record into record[0..3] (HOST memory, 4
 * unsigned, may be NULL): record[0] the bits, record[1] the site of the first
 * failed index check (0: none; 1..5 the GEMV's weight copy, activation copy,
 * output store, partial slots and batch counters; 16..19 attention's K / V
 * copy, query load, output store and split states; 32 the K/V append; 255
 * the self-test below), record[2] / record[3] the low / high word of the
 * offending index (a byte offset for copies, an element or row index
 * otherwise).
 */
q4d_status q4d_device_error_record(unsigned* record, int reset);

/* ------------------------------------------------------ debug build --
 * libq4dec_debug.so is the same library built with Q4D_DEBUG: every global
 * access of every kernel (bulk copies of weights, activations, K and V;
 * query loads; output, partial-slot, state and cache stores; batch counter
 * loads) is first checked against its buffer's extent.  A failed check never
 * traps: it sets bit 2 of the device error record (site and index of the
 * first failure), skips the access or redirects a copy to its buffer's first
 * bytes, and the kernel runs to its end; results of that launch are void.
 * Every compute entry point of the debug build also waits for its stream
 * and returns Q4D_ERR_DEVICE_INDEX or Q4D_ERR_DEVICE_TIMEOUT while the record
 * is set (it stays set until q4d_device_error(1) clears it); on a stream that
 * is being captured into a graph it does not wait.
 * No counterpart in the source pages: a test facility of this library.
 *
 * q4d_debug_build: 1 in the debug build, 0 otherwise.
 * q4d_debug_limit_weights: the GEMV launches and batch descriptors prepared
 *   after this call declare each matrix's weight extent as min(true extent,
 *   bytes) (0: the true extent), so that a test can make the weight-copy
 *   check fail on memory that exists.  Debug build: Q4D_OK.  Release build:
 *   Q4D_ERR_INVALID_ARG, nothing changes.
 * q4d_index_check_selftest: one CTA of 64 threads, the first n_fail of which
 *   (0..64) fail a check with site 255 and index base + thread into the
 *   caller's record (DEVICE pointer to 4 unsigned, 4-byte aligned, zeroed by
 *   the caller); a check that does not return its own condition ORs 4 into
 *   record[0].  Runs in both builds.  Returns Q4D_ERR_INVALID_ARG /
 *   Q4D_ERR_MISALIGNED (nothing launched) or the launch status.
 */
int q4d_debug_build(void);
q4d_status q4d_debug_limit_weights(unsigned long long bytes);
q4d_status q4d_index_check_selftest(unsigned* record, long long base, int n_fail, void* stream);

/* Self-test of the bounded in-kernel wait (the mechanism behind
 * Q4D_ERR_DEVICE_TIMEOUT), for failure-detection tests: one CTA waits on an
 * mbarrier phase that completes only if `arrive` != 0, giving up after
 * limit_us microseconds of wall-clock time.  The kernel ORs 2u into *word if
 * the phase completed and 1u if the wait ran out, then returns normally (the
 * CUDA context stays usable).
 *   word     : device pointer to one unsigned, 4-byte aligned, caller-owned.
 *   limit_us : 1 .. 10,000,000.
 * Returns Q4D_ERR_INVALID_ARG / Q4D_ERR_MISALIGNED (nothing launched) or the
 * launch status; the result is in *word after the stream synchronises.
 * No counterpart in the source pages: a test hook of this library.
 */
q4d_status q4d_wait_selftest(unsigned* word, unsigned limit_us, int arrive, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4DEC_H */
