/*
 * tq.h -- TurboQuant hot path for NVIDIA B200 (sm_100a): C ABI of libtq.so
 *
 * TurboQuant quantizes each key / value vector online and without calibration data:
 * it stores the vector's norm, rotates its direction by a fixed random orthogonal
 * matrix Pi, rounds each rotated coordinate to a Lloyd-Max codebook fitted to the
 * Beta-type coordinate density, and (for keys) adds a 1-bit QJL sign sketch of the
 * residual so that inner products are estimated without bias.  Attention and
 * vector search then read the packed codes directly.
 *
 * Sources cited below:
 *   [ZX]  zingnex.cn thread "TurboQuant：接近理论极限的KV缓存量化方案" -- sections
 *         "随机旋转与Beta分布", "两阶段内积量化".
 *   [TQN] turboquant.net landing page -- sections "PolarQuant：极坐标变换 / 坐标分布公式",
 *         "伪代码实现步骤" (预计算 Lloyd-Max 质心, 生成随机旋转矩阵, Quant / DeQuant 函数,
 *         集成到 Attention), "潜在挑战与解决方案" (随机旋转开销, 残差 norm 存储).
 *   [ADM] admirer.cn news article on Google Research's TurboQuant -- paragraphs on
 *         PolarQuant, QJL, the b-1 + 1 bit two-stage pipeline, vector search.
 *
 * Conventions shared by every call
 *   - All data buffers are owned by the caller; pointers marked "device" must be CUDA
 *     device (or managed) memory on the context's device, "host" pointers host memory.
 *   - Calls never allocate device memory except tq_init (which owns the context's
 *     parameter buffers).  Scratch space is passed in as a caller-owned workspace
 *     whose size is given by the matching *_workspace_size query.
 *   - Every call returns a status (TQ_OK or a TQ_ERR_* code) and never aborts.  On
 *     error, tq_last_error() returns a message for the calling thread.  Kernels are
 *     launched asynchronously on the given stream (NULL = legacy default stream);
 *     execution errors surface at the caller's next synchronisation.
 *   - A context is immutable after tq_init and may be used from several threads and
 *     streams at once.
 *   - The library sets its kernels' shared-memory attributes on a device once and
 *     remembers that it did: after a cudaDeviceReset of that device, load a fresh process
 *     before calling the library on it again.
 *
 * Packed code layout (produced by tq_quantize_kv, read by every other call)
 *   A context with dimension d, MSE bits k (k = bits-1 in prod mode, k = bits in MSE
 *   mode) stores each vector as
 *     - a P-bit code per coordinate, P = k+1 in prod mode, P = k in MSE mode, packed
 *       into code_bytes = P*d_pad/8 bytes with d_pad = 32*ceil(d/32);
 *     - fp16 norm ||x|| (and, prod mode, fp16 residual norm ||r||) in separate arrays.
 *   Code of coordinate i.  With K = 2^k levels (centroids sorted ascending, c[K-1-j] =
 *   -c[j]) the index idx_i of rotated coordinate y_i is stored in sign-magnitude form:
 *   bit k-1 is the negative-half flag n = [idx < K/2], bits 0..k-2 the magnitude rank
 *   m = n ? K/2-1-idx : idx-K/2 (so c[idx] = (n ? -1 : +1) * c[K/2+m]).  For k = 1 the
 *   code is n alone.  In prod mode bit k holds the QJL sign s_i = [(S r)_i >= 0].  Bit
 *   P-1 is called the top bit.
 *   Record.  d_pad/32 groups of P little-endian 32-bit words; group g holds coordinates
 *   32g .. 32g+31.  Inside a group, coordinate e = 8s + j (slice s = 0..3, j = 4h + t
 *   with half h = 0..1, t = 0..3) keeps code bit b at (word, bit):
 *       P = 1:  top        -> (0, E)          E = 8t + 7 - (2s + h)
 *       P = 2:  bit 0      -> (0, 4j + s);                     top -> (1, E)
 *       P = 3:  bits 0, 1  -> (s & 1, 4j + 2*(s >> 1) + b);    top -> (2, E)
 *       P = 4:  bits 0..2  -> (s, 4j + b);   top -> (s, 8t + 7) if h = 0, (s, 8t + 3) if h = 1
 *       P = 5:  bits 0..3 as for P = 4 (bit 3 in the P = 4 top place);  top -> (4, E)
 *   This places, for every slice, the low code bits of four consecutive coordinates as
 *   nibbles of one 16-bit half-word and their top bits as the most significant bits of
 *   four bytes (after one left shift), which is what the decode kernels' byte-permute
 *   table lookups consume.  Coordinates i >= d have code 0.  Slot t of a tq_packed buffer
 *   starts at codes + t*code_bytes.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_ctx tq_ctx;
/* Same type as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st* tq_stream_t;

enum tq_mode {
  TQ_MODE_PROD = 0, /* keys: (bits-1)-bit MSE codebook + 1-bit QJL sign of the residual, m = d */
  TQ_MODE_MSE = 1   /* values: bits-bit MSE codebook only */
};

enum tq_dtype { TQ_DTYPE_F32 = 0, TQ_DTYPE_BF16 = 1, TQ_DTYPE_F16 = 2 };

enum tq_status {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, mismatched contexts, bad dtype */
  TQ_ERR_UNSUPPORTED = 2, /* d or bits outside the supported range, misaligned pointer */
  TQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  TQ_ERR_ALLOC = 4,       /* tq_init could not allocate host or device memory */
  TQ_ERR_WORKSPACE = 5,   /* workspace pointer null or smaller than the size query */
  TQ_ERR_INTERNAL = 6     /* a kernel's own consistency check failed */
};

/* Caller-owned device storage for packed vectors (one context's codes). */
typedef struct tq_packed {
  uint8_t* codes;  /* device [cap][code_bytes]; must be 16-byte aligned */
  uint16_t* norm;  /* device [cap] fp16 bit patterns of ||x|| */
  uint16_t* rnorm; /* device [cap] fp16 bit patterns of ||r||; prod mode only (NULL in MSE mode) */
  int64_t cap;     /* number of slots */
} tq_packed;

/* Static description of a context. */
typedef struct tq_info {
  int d;          /* vector (or channel-group) dimension */
  int bits;       /* total bits per coordinate */
  int k;          /* MSE index bits: bits-1 (prod) or bits (MSE) */
  int m;          /* QJL projection rows (= d in prod mode, 0 in MSE mode) */
  int mode;       /* TQ_MODE_* */
  int planes;     /* P: code bits per coordinate */
  int d_pad;      /* 32*ceil(d/32) */
  int code_bytes; /* P*d_pad/8 */
  uint64_t seed;
} tq_info;

/* tq_init -- build a context: Pi, S, M = S Pi^T and the Lloyd-Max codebook, on the
 * current CUDA device.  [TQN] "生成随机旋转矩阵" (Pi from the QR of a seeded Gaussian
 * d x d matrix, column signs fixed so that R_ii > 0), "预计算 Lloyd-Max 质心" (codebook of
 * 2^k levels on f_d(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-x^2)^((d-3)/2), computed
 * once), [TQN] "随机旋转开销" (generate once, reuse); [ADM] two-stage pipeline (b-1 MSE
 * bits + 1 QJL bit; Gaussian S with m = d rows).
 * Random draws: SplitMix64 seeded with `seed` (output i = mix(seed + (i+1)*0x9E3779B97F4A7C15)),
 * uniforms ((w>>11)+1)*2^-53, Box-Muller pairs (cos, sin); G (d x d, row-major) first,
 * then S (d x d, row-major).
 * Arguments: d in [3, 4096]; bits in [2, 5] (prod) or [1, 4] (MSE); mode TQ_MODE_*.
 * On success *out owns host and device memory released by tq_free.
 * Errors: TQ_ERR_INVALID_ARG (out NULL, bad mode), TQ_ERR_UNSUPPORTED (d or bits out of
 * range), TQ_ERR_ALLOC, TQ_ERR_CUDA. */
int tq_init(tq_ctx** out, int d, int bits, uint64_t seed, int mode);

/* tq_host_params -- the same parameters as tq_init, computed on the host only (no CUDA
 * device needed), for verification.  Output pointers as in tq_get_params (any may be NULL).
 * Errors: as tq_init's argument checks. */
int tq_host_params(int d, int bits, uint64_t seed, int mode, double* Pi, double* S, double* centroids,
                   double* boundaries);

/* Release a context (NULL is ignored).  The caller must ensure no work using it is
 * still queued on any stream. */
void tq_free(tq_ctx* ctx);

/* Kernel-side failure report.  Kernels record the first failure they meet in the
 * context's device error word and carry on or wind down instead of faulting or hanging:
 *   101-109  fused quantize kernel: a pipeline wait exceeded its limit (2 s)
 *   201-203  decode attention: a pipeline wait exceeded its limit
 *   301-305  dequantize: a pipeline wait exceeded its limit (tq_debug_set_wait_limit; 305:
 *            the stall injected by tq_debug_inject_stall)
 *   401-404  workspace quantize path: a pipeline wait exceeded its limit (idem)
 *   501-506  search: a pipeline wait exceeded its limit (idem)
 *   901      a device slot array (dst_slot / src_slot) held a slot outside [0, cap): that
 *            row was skipped (quantize) or written as zeros (dequantize)
 *   902      a channel permutation or column map held an entry out of range: that element
 *            was read as 0 or not written
 * A kernel whose wait gives up drains its in-flight copies and MMAs, releases its tensor
 * memory and returns, so the context stays usable.  This call synchronises the device,
 * copies the word to *code (0 = no failure) and clears it. */
int tq_get_device_error(const tq_ctx* ctx, int* code);

/* Fill *info (host pointer). */
int tq_get_info(const tq_ctx* ctx, tq_info* info);

/* Host float64 copies of the parameters, for verification.  Any pointer may be NULL.
 * Pi [d*d] row-major (y = Pi x), S [m*d] row-major (prod mode; zero rows in MSE
 * mode are not written), centroids [2^k] ascending, boundaries [2^k - 1]. */
int tq_get_params(const tq_ctx* ctx, double* Pi, double* S, double* centroids, double* boundaries);

/* tq_quantize_kv -- quantize n vectors.  [TQN] "Quant / DeQuant 函数" (y = Pi x, nearest
 * centroid per coordinate), "PolarQuant：极坐标变换" (norm stored, direction quantized),
 * "残差 norm 存储" (||r|| as one fp16), [ADM] QJL paragraph (sign of S r).
 * Per vector x (row v of the input):
 *   norm = fp16_rn(||x||); y = Pi x / ||x||; idx_i = #{j : y_i > t_j};
 *   prod mode: r = y - c[idx] (rotated residual; ||r|| equals ||x/||x|| - Pi^T c[idx]||),
 *              rnorm = fp16_rn(||r||), s = [ M r >= 0 ] with M = S Pi^T (= S (x/||x|| - Pi^T c[idx])).
 *   A zero vector stores norm = rnorm = 0, the index of y = 0 and all signs 1.
 * x: device, n rows of d elements of x_dtype (TQ_DTYPE_F32 / BF16 / F16), row v at
 *    x + v*ld elements; ld >= d.  Any channel slice of a wider row is passed by offsetting x.
 * dst: packed storage; vector v goes to slot dst_slot[v] (device int64 array) or, when
 *    dst_slot is NULL, to slot v.  Every slot must be < dst->cap.
 * Kernels: bf16 input with d in {64, 128}, n >= 128, x and ld*2 16-byte aligned runs one
 *    fused tensor-core kernel that needs no workspace.  Every other call runs the
 *    workspace path (a norm / fp16-split kernel, then the rotation GEMM with the
 *    nearest-centroid epilogue and, in prod mode, the QJL GEMM with the sign epilogue,
 *    all on the tensor cores) over row chunks of at most 131072 vectors.
 * workspace: device, 256-byte aligned, >= tq_quantize_workspace_size(ctx, x_dtype, n, ld)
 *    bytes (may be NULL when that size is 0).
 * Errors: TQ_ERR_INVALID_ARG (NULL pointers, n < 0, ld < d, rnorm NULL in prod mode),
 * TQ_ERR_UNSUPPORTED (misaligned codes or workspace), TQ_ERR_WORKSPACE (workspace too
 * small for the path the call takes, e.g. a bf16 x that is not 16-byte aligned), TQ_ERR_CUDA. */
size_t tq_quantize_workspace_size(const tq_ctx* ctx, int x_dtype, int64_t n, int64_t ld);
int tq_quantize_kv(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld,
                   const tq_packed* dst, const int64_t* dst_slot, void* workspace, size_t ws_bytes,
                   tq_stream_t stream);

/* tq_quantize_kv_cols -- tq_quantize_kv of a column subset of each row: element j of vector v
 * is x[v*ld + cols[j]] (cols: device int32 [d], each in [0, ld)), e.g. the channels of one
 * group under an outlier-aware channel permutation (tq_decode_attention_perm).  Runs the
 * workspace path; workspace >= tq_quantize_cols_workspace_size(ctx, n) bytes.  An entry of
 * cols outside [0, ld) reads as 0 and is reported as device error 902.  Errors as
 * tq_quantize_kv, plus TQ_ERR_INVALID_ARG for a NULL cols. */
size_t tq_quantize_cols_workspace_size(const tq_ctx* ctx, int64_t n);
int tq_quantize_kv_cols(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld,
                        const int32_t* cols, const tq_packed* dst, const int64_t* dst_slot, void* workspace,
                        size_t ws_bytes, tq_stream_t stream);

/* tq_dequantize -- MSE reconstruction x_hat = norm * Pi^T c[idx] of n stored vectors
 * ([TQN] "Quant / DeQuant 函数"), one tensor-core GEMM per 128 vectors (centroids as fp16
 * hi + lo against Pi^T as fp16 hi + lo, fp32 accumulation).  Vector v is read from slot
 * src_slot[v] (device int64) or slot v when src_slot is NULL, and written to out + v*ld
 * (device float32, ld >= d).  Prod-mode codes are reconstructed from their index bits.
 * Errors: TQ_ERR_INVALID_ARG (NULL pointers, n < 0, ld < d), TQ_ERR_UNSUPPORTED (d > 128),
 * TQ_ERR_CUDA. */
int tq_dequantize(const tq_ctx* ctx, const tq_packed* src, const int64_t* src_slot, int64_t n,
                  float* out, int64_t ld, tq_stream_t stream);

/* tq_dequantize_qjl -- QJL-augmented reconstruction of stored keys (prod mode):
 *   x_hat = norm * ( Pi^T c[idx] + sqrt(pi/2)/m * rnorm * S^T (2 s - 1) ),
 * the vector whose inner product with any q is the unbiased estimate of tq_attn_logits
 * ([ZX] "两阶段内积量化", [ADM] QJL paragraph: the estimator in vector form).  One
 * tensor-core GEMM per 128 vectors: the centroid part as for tq_dequantize plus the sign
 * part (+-rnorm, exact in fp16, against 16 sqrt(pi/2)/m S^T as fp16 hi + lo).  Arguments,
 * layout and errors as tq_dequantize; TQ_ERR_INVALID_ARG for an MSE-mode context. */
int tq_dequantize_qjl(const tq_ctx* ctx, const tq_packed* src, const int64_t* src_slot, int64_t n,
                      float* out, int64_t ld, tq_stream_t stream);

/* tq_prepare_queries -- rotate queries once: out[a] = (Pi q_a [d floats], S q_a [m floats])
 * ([TQN] "集成到 Attention": the query side of the QJL estimate).  q: device float32
 * [nq][ld]; out: device float32 [nq][d + m]. */
int tq_prepare_queries(const tq_ctx* ctx, const float* q, int64_t nq, int64_t ld, float* out,
                       tq_stream_t stream);

/* tq_attn_logits -- estimated inner products of nq queries with the keys in slots
 * 0..n-1 ([ADM] "computing attention logits" on 4-bit keys; [ZX] "两阶段内积量化"):
 *   logits[a*n + b] = norm_b * ( <Pi q_a, c[idx_b]> + sqrt(pi/2)/m * rnorm_b * <S q_a, 2 s_b - 1> )
 * (prod mode; MSE-mode contexts give the first term only).  q: device float32 [nq][d];
 * logits: device float32 [nq][n].  workspace: device, 16-byte aligned (else TQ_ERR_INVALID_ARG),
 * >= tq_attn_logits_workspace_size. */
size_t tq_attn_logits_workspace_size(const tq_ctx* ctx, int64_t nq);
int tq_attn_logits(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n,
                   float* logits, void* workspace, size_t ws_bytes, tq_stream_t stream);

/* tq_decode_attention -- one decode step of attention over a quantized KV cache
 * ([TQN] "集成到 Attention": k_quant / v_quant replace the cache, QJL estimates <q,k>;
 *  values are MSE-dequantized):
 *   for batch b, query head h (kv head h / (Hq/Hkv)), tokens t < seq_lens[b]:
 *     l_t = scale * sum_g est_g(q[b,h, group g], key g of token t)
 *     out[b,h,:] = sum_t softmax(l)_t * v_hat_t,  v_hat_t[group g] = vnorm * Pi_vg^T c_vg[idx]
 * Channel group g covers channels [group_off[g], group_off[g+1]) of the head dimension D;
 * kctx[g] (prod) and vctx[g] (MSE) must have d = group width.  kcache[g] / vcache[g]
 * hold slot ((b*Hkv + hk)*max_len + t) for token t of sequence b, kv head hk.
 * q: device [B][Hq][D] of q_dtype (F32 or BF16); seq_lens: device int32 [B], each in
 * [0, max_len] (a sequence of length 0 gives zeros); out: device float32 [B][Hq][D].
 * group_off is a host array of ngroups+1 ints with group_off[0] = 0, group_off[ngroups] = D.
 * Hq must be a multiple of Hkv.  workspace: device, >= tq_decode_workspace_size. */
size_t tq_decode_workspace_size(int B, int Hq, int Hkv, int D, int ngroups, int64_t max_len);
int tq_decode_attention(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off,
                        int ngroups, const void* q, int q_dtype, const tq_packed* kcache,
                        const tq_packed* vcache, const int32_t* seq_lens, int B, int Hq, int Hkv,
                        int D, int64_t max_len, float scale, float* out, void* workspace,
                        size_t ws_bytes, tq_stream_t stream);

/* Options of tq_decode_attention_ex (zero / NULL fields keep the defaults).
 * channel_perm -- device int32 [Hkv][D], each row a permutation of 0..D-1: channel group g
 *   of kv head hk covers channels channel_perm[hk*D + group_off[g]] ..
 *   channel_perm[hk*D + group_off[g+1] - 1] of q, K, V and out (the keys and values must
 *   have been quantized with the same columns, e.g. by tq_quantize_kv_cols).  This is how
 *   outlier channels are sent to the higher-bit group of a 2.5 / 3.5-bit split ([ZX]
 *   "KV缓存量化的质量表现": 2.5 and 3.5 bits per channel; turboquant.net "潜在挑战与解决方案":
 *   outlier handling).  NULL: the identity.  An entry outside [0, D) is skipped and
 *   reported as device error 902.
 * block_table, page_tokens -- paged caches ([TQN] "集成到 Attention": the quantized cache
 *   replaces the KV storage of a serving engine; the paging itself is not on the pages):
 *   block_table is device int32 [B][max_len / page_tokens]; token t of sequence b lives in
 *   physical page p = block_table[b][t / page_tokens], and page p of a cache holds kv head
 *   hk's tokens in slots (p*Hkv + hk)*page_tokens .. + page_tokens - 1 (so every cache's
 *   capacity is a whole number of pages of Hkv*page_tokens slots).  page_tokens must be a
 *   positive multiple of 64 dividing max_len.  A page index outside the caches reads page 0
 *   and is reported as device error 901.  NULL: the contiguous layout of
 *   tq_decode_attention. */
typedef struct tq_decode_opts {
  const int32_t* channel_perm;
  const int32_t* block_table;
  int page_tokens;
} tq_decode_opts;

/* tq_decode_attention_ex -- tq_decode_attention with options (opts may be NULL).  Other
 * arguments, layout and errors as tq_decode_attention, except that a paged call only needs
 * caches of at least one page; TQ_ERR_INVALID_ARG for a bad page_tokens. */
int tq_decode_attention_ex(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off,
                           int ngroups, const void* q, int q_dtype, const tq_packed* kcache,
                           const tq_packed* vcache, const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                           int64_t max_len, float scale, float* out, const tq_decode_opts* opts,
                           void* workspace, size_t ws_bytes, tq_stream_t stream);

/* tq_channel_perm_by_score -- host helper for the outlier-aware channel grouping: perm (host
 * int32 [D]) lists the w0 channels with the highest score (ties to the lower channel) in
 * ascending order, then the other channels in ascending order.  With score = a per-channel
 * magnitude statistic of a calibration sample (e.g. the RMS over tokens), declared or
 * detected outlier channels land in the first (higher-bit) group of width w0.  score: host
 * float [D].  Errors: TQ_ERR_INVALID_ARG (NULL pointers, D <= 0, w0 outside [0, D]). */
int tq_channel_perm_by_score(const float* score, int D, int w0, int32_t* perm);

/* Size in bytes of the library-owned scratch array used by tq_decode_attention_static. */
#define TQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)8 << 20)

/* tq_decode_attention_static -- tq_decode_attention for callers that cannot allocate
 * device memory.  The pages have no counterpart to this call; it exists for callers such
 * as plug-ins hosted by an engine that owns all device memory through its own pool, or
 * latency-critical serving loops that may not call cudaMalloc (which can synchronise
 * the device) on the decode path.  Such a caller passes only inputs and outputs; the
 * split-K scratch (prepared queries, per-split softmax partials) lives in a fixed array of
 * TQ_DECODE_STATIC_SCRATCH_BYTES bytes in this library's device memory, which every GPU
 * that loads the library holds until the process exits.  The call allocates nothing.
 * Arguments, layout and results are those of tq_decode_attention.
 * Set-up: the first call on each device (with that device current) looks up the array's
 * device address once and caches it; make that first call before any stream capture.  The
 * cached address does not survive a cudaDeviceReset of that device: do not call this
 * function again in a process after resetting the device.
 * Shared state: every call uses the same array and leaves its contents behind; nothing in
 * it needs to start at zero.  Calls whose GPU work overlaps (on different streams, or
 * from different host threads) race on the array, so serialise them.
 * Errors: first every argument error of tq_decode_attention (TQ_ERR_INVALID_ARG,
 * TQ_ERR_UNSUPPORTED), then TQ_ERR_WORKSPACE when the shape needs more scratch than the
 * array holds (tq_decode_workspace_size > TQ_DECODE_STATIC_SCRATCH_BYTES; use
 * tq_decode_attention with a caller workspace instead), then TQ_ERR_CUDA.  A rejected call
 * launches nothing. */
int tq_decode_attention_static(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off,
                               int ngroups, const void* q, int q_dtype, const tq_packed* kcache,
                               const tq_packed* vcache, const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                               int64_t max_len, float scale, float* out, tq_stream_t stream);

/* tq_search_topk -- top-k stored vectors (slots 0..N-1) of each query by the estimated
 * inner product ([TQN] "向量搜索中的应用"; [ADM] vector-search paragraph).  Ties keep the
 * lower id first.  q: device float32 [nq][d]; scores: device float32 [nq][k] (descending);
 * ids: device int64 [nq][k].  1 <= k <= 64, k <= N.
 * workspace: device, >= tq_search_workspace_size(ctx, nq, N, k).
 * Speed: with q 16-byte aligned and d a multiple of 8 the query projection runs as a
 * register-blocked product; any other q gives the same results through a slower tiled one. */
size_t tq_search_workspace_size(const tq_ctx* ctx, int64_t nq, int64_t N, int k);
int tq_search_topk(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N,
                   int k, float* scores, int64_t* ids, void* workspace, size_t ws_bytes,
                   tq_stream_t stream);

/* Test hooks (not for production use).
 * tq_debug_set_wait_limit -- limit, in nanoseconds, of the pipeline waits of the
 *   dequantize, search and workspace-quantize kernels launched after the call (default 2 s;
 *   0 makes every wait that is not already satisfied give up at once).  Their final
 *   drains of in-flight copies and MMAs keep the 2 s limit, so a kernel that gives up still
 *   leaves no transfer behind.  Process-wide; not thread-safe against concurrent launches.
 * tq_debug_inject_stall -- while on, the dequantize kernel's MMA issuer first waits on a
 *   barrier that nothing arrives on; the wait gives up after the pipeline wait limit,
 *   records device error 305 and the kernel winds down (its output is then undefined).
 * tq_debug_fail_alloc -- make device allocation number `index` (0-based, counted from this
 *   call) inside tq_init fail as if the device were out of memory; -1 disables.  tq_init
 *   then returns TQ_ERR_ALLOC having released everything it allocated. */
int tq_debug_set_wait_limit(uint64_t ns);
int tq_debug_inject_stall(int on);
int tq_debug_fail_alloc(int index);

/* Message describing the calling thread's most recent error ("" if none). */
const char* tq_last_error(void);

/* Number of kernels this library has launched in this process (all streams). */
uint64_t tq_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
