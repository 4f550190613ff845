/*
 * jvp_attn.h -- C ABI of the B200 (sm_100a) masked attention JVP library.
 *
 * Operation (Causal-rCM tech report, Appendix B "FlashAttention-2 JVP Kernel
 * with Custom Masks", Eq. 42-45): for every (batch b, head h) and query row i,
 * with A_i the keys the temporal mask admits for i and c the softmax scale,
 *
 *   O_i   = sum_{j in A_i} p_ij V_j,      p_i = softmax_j( c <Q_i, K_j> )
 *   dS_ij = c ( <dQ_i, K_j> + <Q_i, dK_j> )                     (Eq. 43)
 *   dO_i  = sum_j p_ij (dS_ij - mu_i) V_j + sum_j p_ij dV_j,
 *   mu_i  = sum_j p_ij dS_ij                                     (Eq. 44)
 *   LSE_i = log sum_{j in A_i} exp(c <Q_i, K_j>)
 *
 * i.e. the primal attention output and its forward-mode tangent along
 * (dQ, dK, dV), computed in one streaming pass. The mask has no tangent.
 *
 * Masks (jvp_mask_desc): the token sequence is frame-major with
 * tokens_per_frame (T) tokens per frame, spatial attention within a frame
 * always full; a chunk is `chunk` consecutive frames (the last may be short).
 *   DENSE            L = F*T, every key.
 *   FRAME_CAUSAL     L = F*T, key frame <= query frame (report Sec. 4.1 c1-1).
 *   CHUNK_CAUSAL     L = F*T, key chunk <= query chunk: full inside a chunk,
 *                    causal across chunks (report Sec. 2.3, block-causal).
 *   TEACHER_FORCING  L = 2*F*T, sequence [clean ; noisy] (report Sec. 3.1.1,
 *                    Eq. 8 and Table 2 notes). Clean queries see clean keys
 *                    of chunks <= theirs; noisy queries see clean keys of
 *                    chunks strictly before theirs plus the noisy keys of
 *                    their own chunk.
 * The library turns the descriptor into per-query-tile lists of admissible
 * key tiles (report Appendix B, "Sparse custom-mask representation") and
 * never materialises an L x L mask.
 *
 * Conventions for every call:
 *  - Return 0 (JVP_OK) on success, a negative JVP_ERR_* code otherwise. No
 *    C++ exception crosses this boundary. jvp_attn_strerror() names a code.
 *  - Tensor pointers are caller-owned DEVICE memory on the current CUDA
 *    device, contiguous row-major [B, H, L, d] (lse: [B, H, L] float32),
 *    16-byte aligned. The library keeps no reference after the call returns.
 *  - Launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). Errors detected on the host are returned before any
 *    launch; a kernel that gives up on a bounded wait records a device error
 *    word, read by jvp_attn_check_device_error().
 */
#ifndef JVP_ATTN_H
#define JVP_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define JVP_ATTN_VERSION 100 /* 1.0.0 */

/* ---- error codes --------------------------------------------------------- */
#define JVP_OK                         0
#define JVP_ERR_INVALID_ARG           -1  /* null pointer, bad mode, B/H/L/d <= 0 */
#define JVP_ERR_SHAPE_MISMATCH        -2  /* L inconsistent with the mask descriptor */
#define JVP_ERR_UNSUPPORTED_HEAD_DIM  -3  /* see jvp_attn_fwd for supported d */
#define JVP_ERR_MISALIGNED            -4  /* a tensor pointer not 16-byte aligned */
#define JVP_ERR_LAUNCH_FAILED         -5  /* CUDA launch / runtime error */
#define JVP_ERR_DEVICE_TIMEOUT        -6  /* a kernel gave up on a bounded wait */
#define JVP_ERR_DEVICE_BOUNDS         -7  /* a kernel saw an out-of-range tile index */
#define JVP_ERR_OUT_OF_MEMORY         -8  /* workspace allocation failed */
#define JVP_ERR_UNSUPPORTED_DEVICE    -9  /* current device is not sm_100 */
#define JVP_ERR_TOO_LARGE            -10  /* sizes overflow the kernel's index range */

/* ---- mask descriptor ------------------------------------------------------ */
typedef enum {
  JVP_MASK_DENSE = 0,
  JVP_MASK_FRAME_CAUSAL = 1,
  JVP_MASK_CHUNK_CAUSAL = 2,
  JVP_MASK_TEACHER_FORCING = 3
} jvp_mask_mode;

typedef struct {
  int32_t mode;             /* jvp_mask_mode */
  int32_t tokens_per_frame; /* T >= 1 */
  int32_t n_frames;         /* F >= 1 (per half for TEACHER_FORCING) */
  int32_t chunk;            /* frames per chunk >= 1; ignored by DENSE and
                               FRAME_CAUSAL (which is chunk = 1) */
} jvp_mask_desc;

typedef enum { JVP_BF16 = 0, JVP_FP32 = 1 } jvp_dtype;

/* Tile classes reported by jvp_attn_tile_classes(). */
#define JVP_TILE_EMPTY   0
#define JVP_TILE_FULL    1
#define JVP_TILE_PARTIAL 2

/* ---- the operation ------------------------------------------------------- */
/*
 * jvp_attn_fwd: O, dO and LSE of masked softmax attention and its JVP
 * (Appendix B, Eq. 42-45 of the Causal-rCM report).
 *
 * q, k, v     primal inputs        [B, H, L, d], dtype `dtype`
 * dq, dk, dv  tangents             [B, H, L, d], dtype `dtype`
 * o, d_o      outputs              [B, H, L, d], dtype `dtype`; every row
 *                                  with index < L is written
 * lse         output               [B, H, L] float32, natural log of the sum
 *                                  of exp(scaled scores) over admitted keys
 * softmax_scale  > 0 uses the value given; <= 0 uses 1/sqrt(d). The same
 *             scale multiplies the score and the score tangent.
 *
 * Supported: dtype JVP_BF16 with d = 128 runs the tcgen05/TMEM tensor-core
 * kernel (bf16 operands, fp32 accumulation, bf16 outputs); JVP_FP32, and
 * JVP_BF16 with d in {32, 64, 96}, run a CUDA-core kernel in fp32
 * arithmetic. Other d give JVP_ERR_UNSUPPORTED_HEAD_DIM. B*H*L must stay
 * below 2^31 rows.
 *
 * Workspace: the admissible tile list for (mask, L) is built on the host
 * on first use, copied into a device buffer the library allocates, and
 * cached per (device, mask, L) until jvp_attn_release(). That first call
 * performs a blocking copy and must not be made during stream capture. The
 * tensor-core kernel also takes work items from a 4-byte counter that the
 * library allocates once per (device, stream) and clears on the stream
 * before each launch.
 *
 * A row whose admissible set is empty (no descriptor of the four modes
 * yields one) gets O = dO = 0 and LSE = -inf.
 */
int jvp_attn_fwd(const void* q, const void* k, const void* v,
                 const void* dq, const void* dk, const void* dv,
                 void* o, void* d_o, float* lse,
                 int B, int H, int L, int d, jvp_dtype dtype,
                 jvp_mask_desc mask, float softmax_scale, void* stream);

/*
 * jvp_attn_fwd_scatter: jvp_attn_fwd whose epilogue performs the output
 * exchange of Ulysses context parallelism (Causal-rCM report, Sec. 3.2.1
 * "Parallelisms" and Sec. 3.2.2 "JVP Ulysses CP"): this rank holds a head
 * group of all L tokens, and each output row is stored directly into the
 * token shard that owns it instead of into a local [B, H, L, d] array that
 * an all-to-all would then redistribute.
 *   q, k, v, dq, dk, dv  this rank's head group [B, H, L, d], bf16, d = 128
 *                        (the tensor-core kernel; anything else returns
 *                        JVP_ERR_UNSUPPORTED_HEAD_DIM).
 *   o_dst, d_o_dst, lse_dst  HOST arrays of n_shards device pointers; entry
 *                        r is token-shard owner r's output, [B, h_total,
 *                        L / n_shards, d] bf16 for O and dO and [B, h_total,
 *                        L / n_shards] float32 for LSE. Row n (0 <= n < L) of
 *                        local head h goes to shard r = n / (L / n_shards),
 *                        row n % (L / n_shards), head h0 + h. An entry may
 *                        point into another GPU's memory (peer access or a
 *                        symmetric-memory mapping set up by the caller); the
 *                        kernel writes it with plain stores. The arrays are
 *                        read during the call only.
 *   1 <= n_shards <= 8, L % n_shards == 0, 0 <= h0, h0 + H <= h_total.
 * Rows of a destination not owned by this head group are left untouched;
 * with every rank's call, each shard receives all h_total heads. Visibility
 * on a peer: after this launch completes on every rank, e.g. after a
 * jvp_attn_signal_barrier enqueued behind it on each rank. Errors as jvp_attn_fwd, plus
 * JVP_ERR_INVALID_ARG for a null or out-of-range shard argument and
 * JVP_ERR_MISALIGNED for a destination not 16-byte aligned.
 */
int jvp_attn_fwd_scatter(const void* q, const void* k, const void* v,
                         const void* dq, const void* dk, const void* dv,
                         void* const* o_dst, void* const* d_o_dst, float* const* lse_dst,
                         int n_shards, int h0, int h_total,
                         int B, int H, int L, int d, jvp_dtype dtype,
                         jvp_mask_desc mask, float softmax_scale, void* stream);

/*
 * jvp_attn_signal_barrier: a barrier of the n_ranks processes (one per GPU)
 * of a context-parallel group, enqueued on `stream`. It brackets the fused
 * output exchange of Ulysses context parallelism (Causal-rCM report, Sec.
 * 3.2.2 "JVP Ulysses CP"), where jvp_attn_fwd_scatter stores rows into
 * other ranks' shards: before the launch no rank may still be reading the
 * shard it will receive, and after it a shard is complete only once every
 * rank's kernel is done.
 *
 * flags       host array of n_ranks device pointers: flags[q] is this
 *             process's address of rank q's n_ranks uint32 flag words
 *             (memory every rank can reach, e.g. symmetric memory), all
 *             zero before the first barrier; 4-byte aligned
 * rank        this process's rank, 0 <= rank < n_ranks <= 8
 * epoch       1 for the first barrier on these flags, then 2, 3, ...; every
 *             rank passes the same sequence
 * Once the work enqueued before it on `stream` is complete, the barrier
 * stores epoch into word `rank` of every rank's flags (release, system
 * scope) and waits (acquire loads) until all words of its own flags have
 * reached epoch; work enqueued after it on `stream` starts only then. The
 * wait is bounded by the limit of jvp_attn_set_wait_limit: a rank that
 * never arrives makes the kernel record JVP_ERR_DEVICE_TIMEOUT (read by
 * jvp_attn_check_device_error) and return. Errors: JVP_ERR_INVALID_ARG for a
 * null or out-of-range argument, JVP_ERR_MISALIGNED, JVP_ERR_LAUNCH_FAILED.
 * Allocates nothing.
 */
int jvp_attn_signal_barrier(uint32_t* const* flags, int n_ranks, int rank, uint32_t epoch,
                            void* stream);

/*
 * jvp_attn_fwd_noalloc: jvp_attn_fwd for callers that cannot allocate
 * device memory. The paper has no counterpart: it is a deployment variant.
 *
 * jvp_attn_fwd allocates (cudaMalloc) a device buffer for the tile work list
 * of every new (mask, L). Some callers cannot accept that: a framework whose
 * device memory all belongs to its own pool or arena, or a deployment that
 * forbids device allocation after start-up (where a cudaMalloc can also
 * synchronise the device at a bad moment). This entry point keeps the
 * work list in a fixed array of the library's own device memory (a
 * file-scope __device__ array of 65,536 int32 = 256 KiB, held on every GPU
 * that loads the library until the process exits) and never calls
 * cudaMalloc, cudaFree or any allocating routine. The caller still passes
 * the inputs and outputs.
 *
 * Arguments, layouts and results are those of jvp_attn_fwd, restricted to
 * the tensor-core configuration: dtype must be JVP_BF16 (else
 * JVP_ERR_INVALID_ARG) and d must be 128 (else
 * JVP_ERR_UNSUPPORTED_HEAD_DIM). A mask whose work list needs more than
 * 65,472 words (4 per 128-row query tile + 2 per key-tile run; about 81
 * words per 1000 tokens for the teacher-forcing mask at 1560 tokens per
 * frame, so roughly 800,000 tokens) returns JVP_ERR_TOO_LARGE before any
 * device work.
 *
 * The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) with that device current. The entry point must not
 * be called while `stream` is capturing (it returns JVP_ERR_INVALID_ARG
 * then): which list the array holds is tracked on the host, so a recorded
 * call would replay against whatever list a later call left there. The
 * array holds the kernel's work-item counter
 * (its first 64 words, cleared on `stream` before every launch) and the work
 * list (the rest). A call whose (mask, L) differs from the list the array
 * holds rewrites the list with an asynchronous copy on `stream`; every word
 * the kernel reads is rewritten or cleared, so no earlier contents matter.
 * All calls on a device share the one array: calls whose work overlaps on
 * the GPU (different streams with no ordering between them) race on it and
 * give wrong results. Order such calls on one stream or synchronise
 * between them.
 */
int jvp_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                         const void* dq, const void* dk, const void* dv,
                         void* o, void* d_o, float* lse,
                         int B, int H, int L, int d, jvp_dtype dtype,
                         jvp_mask_desc mask, float softmax_scale,
                         void* stream);

/*
 * jvp_attn_bwd: gradient of sum <G, O> for O = softmax(c QK^T + M) V, the
 * primal output of jvp_attn_fwd. The consistency loss of the Causal-rCM
 * report is differentiated through the primal output only (the JVP is taken
 * at stop-gradient parameters, report Appendix A, around Eq. 26-28), so a
 * training step pairs jvp_attn_fwd with this backward under the same mask:
 *
 *   P = exp(c QK^T - LSE) on admitted pairs,  D_i = <g_i, o_i>,
 *   dP = G V^T,  dS = P o (dP - D),
 *   g_q = c dS K,  g_k = c dS^T Q,  g_v = P^T G.
 *
 * q, k, v, o, g_o   inputs [B, H, L, d] bf16 (o and lse from jvp_attn_fwd)
 * lse               input [B, H, L] float32 (natural log)
 * g_q, g_k, g_v     outputs [B, H, L, d] bf16; every row < L is written
 * scratch           caller-owned device buffer of scratch_len float32, at
 *                   least jvp_attn_bwd_scratch_len(B, H, L) (else
 *                   JVP_ERR_INVALID_ARG); the first pass writes per-row
 *                   softmax statistics there for the second; contents on
 *                   entry are ignored and on return unspecified
 * Supported: JVP_BF16 with d = 128 (two tcgen05 kernels: a query-stationary
 * pass for g_q and D, then a key-stationary pass for g_k and g_v); other
 * dtypes give JVP_ERR_INVALID_ARG, other d JVP_ERR_UNSUPPORTED_HEAD_DIM.
 * Workspace, streams and errors as for jvp_attn_fwd; the key-stationary
 * work list is cached like the query-stationary one.
 */
int jvp_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                 const void* g_o, const float* lse, void* g_q, void* g_k, void* g_v,
                 float* scratch, int64_t scratch_len, int B, int H, int L, int d,
                 jvp_dtype dtype, jvp_mask_desc mask, float softmax_scale, void* stream);

/*
 * jvp_attn_bwd_scratch_len: float32 elements of scratch jvp_attn_bwd needs,
 * 2 * B * H * ceil(L / 128) * 128; -1 if B, H or L is not positive. Host only.
 */
int64_t jvp_attn_bwd_scratch_len(int B, int H, int L);

/* ---- key/value cache: read-only chunk attention and appends ------------- */
/*
 * jvp_attn_cache_fwd: the read-only forward of causal rollout (Causal-rCM
 * report, Sec. 3.2.1 "KV Cache"): the Lq query rows of the current chunk
 * attend to the first Lk rows of a key/value cache, i.e. the committed
 * prefix the chunk needs followed by the chunk's own keys, which the caller
 * has written at their cache position (jvp_attn_rope_copy). With noisy
 * context (Sec. 3.1.3) the committed rows are those of the last denoising
 * forward; the operation is the same.
 *
 *   o = softmax(c q k[0:Lk]^T) v[0:Lk],  lse = log sum exp(c q k[0:Lk]^T)
 *
 * q        [B, H, Lq, d] bf16            o    [B, H, Lq, d] bf16 (output)
 * k_cache, v_cache [B, H, Lcache, d] bf16 (rows Lk..Lcache-1 are not read;
 *          the kernel's tensor maps stop at Lk)
 * lse      [B, H, Lq] float32, natural log (output)
 * softmax_scale <= 0 selects 1/sqrt(d). Requires 1 <= Lk <= Lcache, Lq >= 1,
 * dtype JVP_BF16 (else JVP_ERR_INVALID_ARG) and d = 128 (else
 * JVP_ERR_UNSUPPORTED_HEAD_DIM); all pointers 16-byte aligned. The
 * (b, h, 128-row query tile) items that fill whole waves of the GPU run
 * whole; the items left over are cut into key ranges spread over the SMs,
 * and a second kernel combines their partial results. The library keeps the
 * partial-result workspace per (device, stream), grows it when a larger
 * call needs it (JVP_ERR_OUT_OF_MEMORY on failure) and frees it in
 * jvp_attn_release. Asynchronous on `stream`; errors as jvp_attn_fwd.
 */
int jvp_attn_cache_fwd(const void* q, const void* k_cache, const void* v_cache, void* o,
                       float* lse, int B, int H, int Lq, int Lk, int Lcache, int d,
                       jvp_dtype dtype, float softmax_scale, void* stream);

/*
 * jvp_attn_rope_copy: copies rows [src_row0, src_row0 + rows) of every
 * (b, h) slice of src [B, H, src_rows, d] to rows [dst_row0, dst_row0 +
 * rows) of dst [B, H, dst_rows, d] (same dtype), optionally rotating them
 * with rotary position embedding (Sec. 3.2.1: post-RoPE caching rotates
 * keys once when they are appended; pre-RoPE caching stores them unrotated
 * and rotates the exposed prefix into a working buffer before a read).
 * With rope_cos and rope_sin (both non-null, float32 [rope_rows, d/2]), row
 * j of the range is rotated by table row rope_row0 + j: each pair
 * (x_2i, x_2i+1) becomes (x_2i c - x_2i+1 s, x_2i s + x_2i+1 c), computed
 * in fp32 and rounded once. Both null: a plain copy (values, or keys of a
 * pre-RoPE cache). src and dst may be the same buffer only with identical
 * row ranges (in place); otherwise the ranges must not overlap.
 * Requires rows >= 0 (0: nothing to do), src_row0 + rows <= src_rows,
 * dst_row0 + rows <= dst_rows, rope_row0 + rows <= rope_rows, d a multiple
 * of 8 (bf16) or 4 (fp32), 16-byte aligned src/dst and tables (else
 * JVP_ERR_INVALID_ARG / JVP_ERR_MISALIGNED). Asynchronous on `stream`.
 */
int jvp_attn_rope_copy(const void* src, void* dst, int B, int H, int src_rows, int dst_rows,
                       int rows, int src_row0, int dst_row0, int d, jvp_dtype dtype,
                       const float* rope_cos, const float* rope_sin, int rope_rows,
                       int rope_row0, void* stream);

/* ---- attention-layer tangent prologue ------------------------------------ */
/*
 * jvp_attn_qkv_prologue: the primal-tangent hand-off from an attention
 * layer's fused QKV projection to jvp_attn_fwd (layer-level JVP, Causal-rCM
 * report Sec. 3.2.2 "JVP FSDP2": each layer maps (x, dx) to (y, dy); with
 * the weights at their stop-gradient values the projection tangent is
 * dx W, computed by the caller's GEMM). For every token, q and k are RMS
 * normalised over groups of norm_group channels with weights norm_q /
 * norm_k, their tangents by the derivative of that normalisation
 *   r = 1/sqrt(mean(a^2) + eps),  y = a r w,  dy = w r (da - a mean(a da) r^2),
 * then both are rotated by rotary position embedding (row l of rope_cos /
 * rope_sin [rope_rows >= L, d/2], float32, pairs (x_2i, x_2i+1) as in
 * jvp_attn_rope_copy; the tangent rotates like the primal), and q, k, v and
 * their tangents are written in the [B, H, L, d] layout of jvp_attn_fwd.
 *
 * qkv, d_qkv   [B, L, 3 H d] bf16: [q | k | v] of x and of dx, each block
 *              H*d channels, channel h*d + j = head h, dimension j
 * q .. dv      outputs [B, H, L, d] bf16
 * norm_q, norm_k  float32 [norm_group], both NULL for no normalisation;
 *              norm_group is H*d (one group per token) or d (per head)
 * rope_cos, rope_sin  both NULL for no rotation
 * Requires dtype JVP_BF16, d a power of two in [8, 256]
 * (else JVP_ERR_UNSUPPORTED_HEAD_DIM), H*d a multiple of 256, 16-byte
 * aligned pointers. Memory-bound; asynchronous on `stream`.
 */
int jvp_attn_qkv_prologue(const void* qkv, const void* d_qkv, void* q, void* k, void* v,
                          void* dq, void* dk, void* dv, const float* norm_q,
                          const float* norm_k, int norm_group, float eps,
                          const float* rope_cos, const float* rope_sin, int rope_rows, int B,
                          int L, int H, int d, jvp_dtype dtype, void* stream);

/* ---- host-side mask / schedule queries (no GPU needed) ------------------- */
/*
 * jvp_attn_mask_stats: for the mask on L tokens and a bm x bn tile grid
 * anchored at (0, 0): *pairs = admitted (query, key) pairs per head;
 * *full / *partial / *empty = number of tiles in which all / some / none of
 * the (query < L, key) slots are admitted. Query rows at or past L are
 * ignored (they are never written); a tile whose key range reaches past L
 * is never full. Any output pointer may be NULL. Host only.
 */
int jvp_attn_mask_stats(jvp_mask_desc mask, int L, int bm, int bn,
                        int64_t* pairs, int64_t* full, int64_t* partial,
                        int64_t* empty);

/*
 * jvp_attn_tile_classes: writes the class (JVP_TILE_*) of every tile of the
 * bm x bn grid to out[qt * n_kt + kt], n_qt = ceil(L/bm), n_kt = ceil(L/bn).
 * out_len must be >= n_qt * n_kt, else JVP_ERR_INVALID_ARG. Host only.
 */
int jvp_attn_tile_classes(jvp_mask_desc mask, int L, int bm, int bn,
                          int8_t* out, int64_t out_len);

/*
 * jvp_attn_schedule: the work list the tensor-core kernel runs, for tests
 * and tools. Query tiles are bm rows; key tiles bn keys. Writes up to
 * qtile_cap entries of 4 int32 {query tile, first segment, segment count,
 * key tiles} to `qtiles`, longest first (ties: lower query tile first), and
 * up to seg_cap segments of 3 int32 {first key tile, key-tile count,
 * partial flag} to `segs`, each query tile's segments in increasing key
 * order. *n_qtiles / *n_segs receive the full counts even if a cap is too
 * small (then JVP_ERR_INVALID_ARG is returned). Host only.
 */
int jvp_attn_schedule(jvp_mask_desc mask, int L, int bm, int bn,
                      int32_t* qtiles, int qtile_cap, int32_t* segs,
                      int seg_cap, int* n_qtiles, int* n_segs);

/*
 * jvp_attn_schedule_kv: the key-tile-major work list of jvp_attn_bwd's key
 * pass, for tests and tools: entries of 4 int32 {key tile, first segment,
 * segment count, query tiles} (key tiles of bk keys with work, longest
 * first) and segments of 3 int32 {first query tile, count, partial flag}
 * over query tiles of bq rows. A tile is full only if all its (query, key)
 * slots are admitted and it reaches past L in neither direction. Caps and
 * counts as for jvp_attn_schedule. Host only.
 */
int jvp_attn_schedule_kv(jvp_mask_desc mask, int L, int bq, int bk,
                         int32_t* ktiles, int ktile_cap, int32_t* segs,
                         int seg_cap, int* n_ktiles, int* n_segs);

/* ---- device error word, workspace, misc ---------------------------------- */
/*
 * jvp_attn_check_device_error: synchronises `stream`, then reads and clears
 * the current device's error word. Returns JVP_OK, JVP_ERR_DEVICE_TIMEOUT,
 * JVP_ERR_DEVICE_BOUNDS, or JVP_ERR_LAUNCH_FAILED if the stream itself
 * reports a CUDA error.
 */
int jvp_attn_check_device_error(void* stream);

/*
 * jvp_attn_set_wait_limit: upper bound, in nanoseconds, on each wait inside
 * the tensor-core kernel (for a pipeline stage, a peer warp or a work item).
 * A wait that runs out makes the kernel record JVP_ERR_DEVICE_TIMEOUT in the
 * device error word, let its own copies and MMAs finish, free its tensor
 * memory and exit; the CUDA context stays usable and the outputs of that
 * launch are undefined. 0 restores the default of 2 s. Process-wide; applies
 * to launches made after the call. A tiny limit is how the failure path is
 * tested without faulting a GPU.
 */
int jvp_attn_set_wait_limit(uint64_t ns);

/*
 * jvp_attn_set_stall_test: failure-detection test switch. While enabled
 * (enable != 0), the MMA warp of every tensor-core kernel launched
 * (attention JVP, both backward passes, cache attention) first waits on a
 * barrier phase that nothing completes, so the wait runs out after the limit
 * set by jvp_attn_set_wait_limit and the launch ends through its timeout
 * path: JVP_ERR_DEVICE_TIMEOUT in the device error word, outputs undefined,
 * context usable. No memory is touched out of bounds and nothing traps.
 * Process-wide; applies to launches made after the call; 0 turns it off.
 * Always returns JVP_OK.
 */
int jvp_attn_set_stall_test(int enable);

/* Frees every cached workspace on every device. Synchronises the device(s)
 * first. Safe to call at any time outside stream capture. */
int jvp_attn_release(void);

/* Static string naming an error code (never NULL). */
const char* jvp_attn_strerror(int code);

/* JVP_ATTN_VERSION of the loaded library. */
int jvp_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JVP_ATTN_H */
