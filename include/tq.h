/*
 * tq.h -- C ABI of libtq: TurboQuant online KV-cache vector quantization and
 * decode attention over the packed cache, for NVIDIA B200 (sm_100a).
 *
 * The method (page "TurboQuant-MLX: quantizzare pesi e KV cache per LLM
 * open-weight su Mac", section "Il metodo TurboQuant, in breve"): each head
 * vector x is rotated by a seeded random orthogonal matrix Pi, every rotated
 * coordinate is quantized on its own to the nearest Lloyd-Max centroid of the
 * known post-rotation coordinate density, and the b-bit codes are packed next
 * to the vector's norm.  The inner-product ("prod") variant spends one of the
 * b bits per channel on a 1-bit QJL sketch sign(S r) of the residual r so that
 * <q, x> is estimated without bias.  No calibration: everything depends only
 * on (d, b, seed).
 *
 * Conventions for every call below
 *  - Memory: the caller owns all memory.  Device pointers are plain CUDA
 *    device addresses (for example from torch tensors); host pointers are
 *    plain host arrays.  No call on the data path allocates; tq_params_create
 *    allocates the parameter tables once and tq_params_destroy frees them.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream).  Device calls only enqueue work and never synchronize.
 *    tq_append and tq_decode_attn may therefore be captured into a CUDA
 *    graph on a capturing stream (tq_append's side stream, used when K and V
 *    formats differ, forks from and joins back into it) once each has been
 *    called eagerly on the device, which sets the kernels' attributes; a
 *    replay reads the lengths on the device, so it appends after and
 *    attends over whatever the cache holds at replay time.
 *  - Errors: every call returns a tq_status; TQ_OK is 0.  On failure nothing
 *    is enqueued and tq_last_error() returns a message for the calling host
 *    thread.  Inputs must be finite: NaN or Inf inputs give unspecified codes
 *    but never an out-of-bounds access.
 *  - Sizes: d = 128 and m = 128 in this version (TQ_ERR_UNSUPPORTED
 *    otherwise); bits in 1..4 or 8 (MSE; 8 = one byte per code, 256
 *    centroids, uniform rows only) or 1..4 total (prod, 1 = QJL only).
 *
 * Packed row format (both sides of the library agree on it; the pages only
 * say that codes live at "unconventional bit widths", NVIDIA forum post "Why
 * TurboQuant saves DGX twice"):
 *  - codes: code j of rotated coordinate j sits at bit offset sum_{i<j} w_i of
 *    the row, least-significant bit first inside little-endian bytes.  w_j is
 *    the MSE bit width (bits for MSE, bits-1 for prod); a mixed row uses
 *    bits+1 for j < d/2.  Row bytes: 16*w (uniform) or 8*(2w+1) (mixed).
 *  - code value = number of Lloyd-Max decision bounds strictly below the
 *    rotated unit-vector coordinate (ties go to the lower centroid).
 *  - norms: fp32 ||x||.  qjl (prod): m/8 bytes per row, bit i = 1 iff
 *    (S r)_i >= 0.  res_norms (prod): fp32 ||r||.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_ARG = 1,          /* NULL pointer, negative size, bad enum */
  TQ_ERR_UNSUPPORTED = 2,  /* a size or format this build does not handle */
  TQ_ERR_ALIGN = 3,        /* a device plane not 16-byte aligned */
  TQ_ERR_CAPACITY = 4,     /* workspace or cache too small */
  TQ_ERR_CUDA = 5,         /* a CUDA runtime call failed (message says which) */
  TQ_ERR_NOMEM = 6         /* tq_params_create could not allocate */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;
typedef enum { TQ_MODE_MSE = 0, TQ_MODE_PROD = 1 } tq_mode;
typedef enum { TQ_K = 0, TQ_V = 1 } tq_which;
typedef enum { TQ_ROT_HAAR = 0, TQ_ROT_HADAMARD = 1 } tq_rotation_kind;

/* Parameters of one quantizer pair (keys and values may differ: the
 * asymmetric K/V setting of "Greetings from TurboQuant-MLX" (turboquant_plus
 * issue 59) and of the TurboQuant-MLX article, section "Cosa aggiunge").
 * bits_*: total bits per channel.  mixed_*: 1 puts the first d/2 rotated
 * channels at bits+1 ("3.5 bits per channel" with bits = 3 and "2.5 bits per
 * channel" with bits = 2, article section "Il metodo TurboQuant, in breve");
 * MSE mode only, bits 2 or 3 (else TQ_ERR_UNSUPPORTED).  seed drives Pi and S. */
typedef struct {
  int d;
  int bits_k, bits_v;
  int mode_k, mode_v;    /* tq_mode */
  int mixed_k, mixed_v;  /* 0 or 1 */
  int m;                 /* QJL sketch size */
  uint64_t seed;
  int rotation;          /* tq_rotation_kind: dense Haar Pi (0) or randomized Hadamard (1) */
} tq_config;

typedef struct tq_params tq_params;

/* One packed plane set (device pointers).  codes: [n][code_bytes];
 * norms: [n] fp32; qjl: [n][m/8] (prod only, else NULL); res_norms: [n] fp32
 * (prod only, else NULL).  Planes must be 16-byte aligned (TQ_ERR_ALIGN). */
typedef struct {
  uint8_t* codes;
  float* norms;
  uint8_t* qjl;
  float* res_norms;
} tq_packed;

/* ---- host tables ------------------------------------------------------ */

/* Lloyd-Max codebook of one coordinate of a uniform point on S^{d-1}
 * (density proportional to (1-x^2)^((d-3)/2)), article section "Il metodo
 * TurboQuant, in breve" (optimal scalar quantizer for the known distribution)
 * and section "Cosa aggiunge turboquant-mlx" (Lloyd-Max).  Writes 2^bits
 * ascending centroids and the 2^bits - 1 midpoints between them (host
 * arrays, caller-owned).  Any d >= 3 and bits in 1..8: up to 4 bits by the
 * plain Lloyd iteration, above by Newton's method on the same conditions
 * (the plain iteration slows down as the levels grow).  Pure host function. */
tq_status tq_codebook(int d, int bits, double* centroids, double* bounds);

/* Seeded random rotation Pi (d x d row-major, y = Pi u): Haar orthogonal,
 * the QR factor of a Gaussian matrix with diag(R) made positive.  Gaussians
 * from SplitMix64 (stream seed ^ (0 << 32)) and Box-Muller, filled row-major.
 * Host array of d*d doubles, caller-owned.  Pure host function. */
tq_status tq_rotation(uint64_t seed, int d, double* pi);

/* Randomized Hadamard rotation, the port's realization of the random rotation
 * (TurboQuant-MLX article, section "Cosa aggiunge turboquant-mlx"):
 * Pi = H D / sqrt(d) with H the Walsh-Hadamard matrix (Sylvester order,
 * H[i][j] = (-1)^popcount(i & j)) and D = diag(s), s_j = -1 when the top bit
 * of SplitMix64 output j of stream seed ^ (2 << 32) is set, else +1.  d a
 * power of two; host array of d*d doubles (row-major, y = Pi u), caller-owned.
 * Pure host function. */
tq_status tq_hadamard_rotation(uint64_t seed, int d, double* pi);

/* QJL matrix S (m x d row-major, i.i.d. N(0,1)) from the stream
 * seed ^ (1 << 32).  Host array of m*d doubles.  Pure host function. */
tq_status tq_qjl_matrix(uint64_t seed, int m, int d, double* s);

/* ---- parameters ------------------------------------------------------- */

/* Build the tables for cfg on the current CUDA device (allocates device
 * memory once, copies with the legacy stream and synchronizes; not for the
 * data path).  *out is owned by the caller and freed by tq_params_destroy. */
tq_status tq_params_create(const tq_config* cfg, tq_params** out);
void tq_params_destroy(tq_params* p);

/* Error bits that tq_quantize kernels recorded on the device for p (appends
 * record into their cache's status word instead): 4 = a wait in the copy /
 * tensor-core pipeline gave up after its time limit (the outputs of that call
 * are invalid).  Copies the word to *out (synchronizing the device); clear != 0
 * then resets it.  Not for the data path. */
tq_status tq_params_status(const tq_params* p, int32_t* out, int clear);

/* Bytes per packed row for K (which = TQ_K) or V: code bytes and QJL bytes
 * (0 in MSE mode). */
tq_status tq_row_bytes(const tq_params* p, int which, int* code_bytes, int* qjl_bytes);

/* ---- quantize / dequantize ------------------------------------------- */

/* Rotate, quantize and pack n vectors x ([n][d], fp32 or bf16, device) with
 * the K or V format of p into `out` (device planes sized for n rows).
 * Article section "Il metodo TurboQuant, in breve".  n = 0 is a no-op.
 * bf16 input (x 16-byte aligned) runs the rotation, and in prod formats the
 * residual sketch, on the tensor cores (tcgen05, the matrices split into two
 * bf16 halves, fp32 accumulation); fp32 input uses an fp32 SIMT kernel. */
tq_status tq_quantize(const tq_params* p, const void* x, int x_dtype, int64_t n, int which,
                      const tq_packed* out, void* stream);

/* x_hat = ||x|| (Pi^T c[idx] + sqrt(pi/2)/m * ||r|| * S^T z) for n packed rows
 * (device) into out ([n][d] fp32, device); accumulates in fp64.  A boundary
 * and test call: decode attention never materializes x_hat. */
tq_status tq_dequantize(const tq_params* p, const tq_packed* in, int64_t n, int which,
                        float* out, void* stream);

/* ---- packed KV cache ---------------------------------------------------- */

/* A cache for n_seq sequences x n_kv_heads heads.  Token t of a sequence is
 * kept unquantized in bf16 if t < n_sink (attention sink, "Greetings from
 * TurboQuant-MLX", item 1) and is quantized row t - n_sink otherwise.
 * capacity is a multiple of 64 and counts quantized rows.  Planes are laid
 * out per unit: [n_seq][n_kv_heads][...] with a unit's data contiguous.
 *  - norms, res_norms: [capacity] fp32; qjl: [capacity][m/8] bytes (row order).
 *  - sink planes: [n_sink][d] bf16.
 *  - code planes (k_codes, v_codes): [capacity / 16] tiles of 16 rows,
 *    16 * code_bytes bytes each, arranged for the decode kernel rather than
 *    in row order.  Write and read them through tq_append,
 *    tq_cache_write_rows and tq_cache_read_rows.  Inside a tile, lane
 *    L = 4g + t (g, t in 0..7, 0..3) of the decoding warp owns a block of
 *    code_bytes / 2 bytes: for keys, of tokens g and g + 8, the bytes of the
 *    packed row holding quarter t of each code segment ([A.seg0 | B.seg0 |
 *    A.seg1 | B.seg1], A = token g, B = token g + 8); for values, of tokens
 *    2t, 2t+1, 2t+8, 2t+9 (a, b, c, d), eighth g of each segment ([a.seg0 |
 *    b.seg0 | c.seg0 | d.seg0 | a.seg1 | ... | d.seg1]).  A segment is the
 *    whole row (uniform widths) or one of its two halves of 64 coordinates
 *    (mixed rows); every such piece is a whole number of bytes.  The blocks
 *    are stored as columns: the first 16 bytes of every lane (lane L's at
 *    offset 16 L), then the next 16 and so on while 16 bytes remain, then 8,
 *    then 4, as the block's size needs.  So each lane reads its share with one load per column and the
 *    warp's loads never share a shared-memory bank.
 * lens: device int32 [n_seq], tokens held per sequence (sink included); the
 * caller zeroes it for an empty cache.  status: device int32 word, zeroed by
 * the caller with the cache; kernels OR error bits into its low 16 bits (1 =
 * append past capacity, 2 = a length above the bound given to
 * tq_decode_attn, 4 = a decode wait on the copy pipeline gave up after its
 * time limit, 8 = the decode kernel's shared-memory layout did not fit; after
 * 4 or 8 the outputs are invalid).  Bits 16..31 count the CTAs of a running
 * tq_append and are zero again when it ends. */
typedef struct {
  int n_seq, n_kv_heads, capacity, n_sink;
  uint8_t* k_codes; float* k_norms; uint8_t* k_qjl; float* k_res_norms;
  uint8_t* v_codes; float* v_norms; uint8_t* v_qjl; float* v_res_norms;
  uint16_t* k_sink; uint16_t* v_sink;
  int32_t* lens;
  int32_t* status;
} tq_cache;

/* Bytes of one contiguous buffer holding every plane of such a cache (each
 * plane 256-byte aligned); 0 on bad arguments. */
size_t tq_cache_bytes(const tq_params* p, int n_seq, int n_kv_heads, int capacity, int n_sink);

/* Fill *out with plane pointers carved from `base` (device, >= tq_cache_bytes
 * bytes, 256-byte aligned).  lens and status are separate caller buffers. */
tq_status tq_cache_bind(const tq_params* p, void* base, size_t bytes, int n_seq, int n_kv_heads,
                        int capacity, int n_sink, int32_t* lens, int32_t* status, tq_cache* out);

/* Append n_tok new tokens to each of n_seq sequences (streaming append,
 * "Greetings from TurboQuant-MLX", item 2: 64-token chunks; the method is
 * online, article section "Il metodo TurboQuant, in breve").  seq_ids:
 * device int32 [n_seq], distinct cache sequence indices.  k, v: device
 * [n_seq][n_tok][n_kv_heads][d] in dtype.  Tokens land at positions
 * lens[s] .. lens[s] + n_tok - 1 (sink or quantized row), then lens[s] grows
 * by n_tok, all in stream order.  A sequence that would pass
 * n_sink + capacity is left unchanged and bit 1 is set in cache->status.
 * When K and V share a format and dtype is bf16 one kernel quantizes both;
 * otherwise the keys' kernel runs on `stream` and the values' on a side
 * stream of the library's, joined back before the call returns.  The CTA that
 * finishes last updates lens (no separate launch), so appends to one cache
 * must not overlap on the GPU. */
tq_status tq_append(const tq_params* p, const tq_cache* cache, const int32_t* seq_ids,
                    const void* k, const void* v, int dtype, int n_tok, int n_seq, void* stream);

/* Copy n packed rows (tq_quantize's row format, device planes `rows`, 16-byte
 * aligned) into quantized rows row0 .. row0 + n - 1 of unit (seq, kv_head) of
 * the cache, K side (which = TQ_K) or V side: codes into the tiled code plane,
 * norms, and in prod mode the QJL rows and residual norms.  lens and the sink
 * are not touched.  For importing rows quantized elsewhere (or by the
 * oracle in tests).  row0 + n > capacity gives TQ_ERR_CAPACITY.
 * Asynchronous on `stream`. */
tq_status tq_cache_write_rows(const tq_params* p, const tq_cache* cache, int which, int seq, int kv_head,
                              int row0, int64_t n, const tq_packed* rows, void* stream);

/* The reverse: quantized rows row0 .. row0 + n - 1 of unit (seq, kv_head)
 * into packed rows (tq_quantize's format).  Asynchronous on `stream`. */
tq_status tq_cache_read_rows(const tq_params* p, const tq_cache* cache, int which, int seq, int kv_head,
                             int row0, int64_t n, const tq_packed* rows, void* stream);

/* ---- decode attention --------------------------------------------------- */

/* sparse_v_threshold: V of a quantized token is left out when an upper bound
 * on its softmax weight is below this value (0 = off); the softmax
 * denominator keeps every token ("Greetings from TurboQuant-MLX", item 3:
 * 1e-6).  The bound used is exp(s - m) / max(l, 1) with m the running maximum
 * of the scores seen so far by the decoding warp and l a partial sum of their
 * weights; it is never below the final weight, so no token the exact rule
 * keeps is skipped.  The value work of a 32-token tile is skipped when all its
 * (token, query head) weights are dropped.
 * sparse_v_stats: NULL, or a device array of 4 uint64 (8-byte aligned) that
 * the call adds its tallies to when sparse V is on (the caller zeroes it):
 * [0] (quantized token, query head) weights examined, [1] weights dropped,
 * [2] 32-token warp tiles examined, [3] tiles whose value work was skipped.
 * reserved must be 0. */
typedef struct {
  float sparse_v_threshold;
  int reserved;
  unsigned long long* sparse_v_stats;
} tq_attn_flags;

/* Workspace bytes for tq_decode_attn on B sequences with n_kv_heads heads,
 * Hq query heads and lengths up to max_len. */
size_t tq_decode_workspace_bytes(const tq_params* p, int B, int hq, int n_kv_heads, int max_len);

/* Zero-fill a workspace.  Optional: the decode kernels keep no state in the
 * workspace between calls and read only what they wrote earlier in the same
 * call. */
tq_status tq_decode_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* One decode step for sequences b = 0..B-1 of the cache: q [B][hq][d]
 * (q_dtype), out [B][hq][d] (out_dtype), GQA: query head h reads kv-head
 * h / (hq / n_kv_heads), hq / n_kv_heads <= 8.  Score <q, k>/sqrt(d) with the
 * key read through its codes: s = ||k|| (<Pi q, c[idx]> + sqrt(pi/2)/m ||r||
 * <S q, z>) / sqrt(d); softmax over all held tokens; V accumulated in the
 * rotated domain and Pi^T (and S^T) applied once per output.  Sink tokens use
 * their bf16 keys and values directly.  A sequence with no tokens gives a
 * zero output.  max_len: host bound on lens (longer sequences are cut to it
 * and bit 2 is set in cache->status).  n_sink above 4096 gives
 * TQ_ERR_UNSUPPORTED.  K/V formats with a decode kernel: equal formats
 * (MSE 1..4 bits, mixed 2.5 and 3.5, prod 1..4) and the asymmetric MSE pairs
 * K4/V3, K4/V2, K3/V2 and K8/V3 (8-bit keys); any other pair gives
 * TQ_ERR_UNSUPPORTED.  Three kernels run on the stream: the
 * query rotation, the persistent decode kernel and the merge, each launched
 * with programmatic stream serialization so that its prologue overlaps the
 * previous kernel's tail; the rotation reads q only after the kernel before
 * it on the stream has finished, so q and the cache may be written by the
 * work just before the call.  Nothing in the workspace needs to start at
 * zero. */
tq_status tq_decode_attn(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache,
                         int B, int hq, int max_len, void* out, int out_dtype,
                         void* workspace, size_t ws_bytes, const tq_attn_flags* flags,
                         void* stream);

/* The same decode step as tq_decode_attn for callers that cannot allocate
 * device memory (for example an engine that reserves all device memory for its
 * own pool and calls this library from plugin code without a handle on that
 * pool, or a decode loop that cannot afford cudaMalloc's implicit device
 * synchronization).  No counterpart in the method's pages: it only changes
 * where the workspace lives.  The workspace is a fixed 8 MiB array in device
 * memory defined by the library (every GPU that loads the library holds it
 * until the process exits); a call that would need more than 8 MiB (see
 * tq_decode_workspace_bytes) returns TQ_ERR_CAPACITY.  Arguments are checked
 * exactly as tq_decode_attn checks them.  No cudaMalloc, cudaFree or other
 * allocation happens.  The first call on each device looks up the array's
 * address (cudaGetSymbolAddress), and so does the first call after the
 * device's context was replaced (cudaDeviceReset); make such a call before any
 * stream capture.  No call clears the array and none needs to: every word a
 * kernel reads was written earlier in the same call.  All calls share the
 * array, so calls that overlap on the GPU (for example on two streams) race. */
tq_status tq_decode_attn_noalloc(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache,
                                 int B, int hq, int max_len, void* out, int out_dtype,
                                 const tq_attn_flags* flags, void* stream);

/* Message for the last failed call on this host thread ("" if none). */
const char* tq_last_error(void);

/* ---- inner-product search ---------------------------------------------- */

/* Workspace bytes of tq_search on the current device (the same for every
 * database size and number of queries). */
size_t tq_search_workspace_bytes(void);

/* Top-k inner-product search over a database of n rows quantized with the
 * `which` format of p (tq_quantize output: device planes, 16-byte aligned),
 * the second application of the quantizer in the TurboQuant-MLX article,
 * section "Il metodo TurboQuant, in breve" (similarity search in place of
 * product quantization).  Row i scores <q_j, x^_i> for query j, the inner
 * product with the row's reconstruction: ||x_i|| (<Pi q_j, c[idx_i]> +
 * sqrt(pi/2)/m ||r_i|| <S q_j, z_i>) in prod mode (the unbiased estimate of
 * <q_j, x_i>), the first term alone in MSE mode.
 *   q:      [n_queries][d] (q_dtype), device, 16-byte aligned.
 *   scores: [n_queries][k] fp32, rows: [n_queries][k] int64, device,
 *           caller-owned: per query the k best rows, larger score first,
 *           equal scores in row order; with n < k the tail holds score -inf
 *           and row -1.
 * Every format tq_params_create accepts is searchable (MSE 1..4 and 8 bits,
 * mixed 2.5 and 3.5, prod 1..4).
 * Scores come from fp16 tensor-core products with fp32 accumulation: rows
 * whose scores differ by less than about 1e-3 of ||q|| ||x|| may come in
 * either order.  1 <= k <= 32 (TQ_ERR_UNSUPPORTED above), 0 <= n < 2^31,
 * n_queries >= 1 (the database is read once per group of 8 queries).
 * workspace: device, >= tq_search_workspace_bytes() bytes, 16-byte aligned;
 * calls sharing it must not overlap.  Asynchronous on `stream`; error bits
 * go to the params status word (tq_params_status). */
tq_status tq_search(const tq_params* p, int which, const tq_packed* db, int64_t n, const void* q, int q_dtype,
                    int n_queries, int k, float* scores, int64_t* rows, void* workspace, size_t ws_bytes,
                    void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
