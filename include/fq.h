/*
 * fq.h - C ABI of the FibQuant KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * FibQuant ("FibQuant: Universal Vector Quantization for Random-Access KV-Cache Compression",
 * technical summary sec. 2.3) encodes a key or value vector x in R^d as
 *   - its norm nu = |x|_2 (stored as IEEE fp16, round to nearest even),
 *   - the unit vector rotated by one shared Haar matrix, z = Pi x / nu,
 *   - split into m = d'/k blocks of k consecutive coordinates, each replaced by the index of
 *     its nearest codeword in one shared codebook of N codewords (B = log2 N bits each).
 * The decoder fetches the codewords, concatenates them, applies Pi^T and scales by nu.
 * Records are fixed-size so that any token decodes alone by address arithmetic (summary
 * sec. 1, "random access").
 *
 * Notation used below:  d = vector length; k = block size; d' = k * ceil(d / k) (x is
 * zero-padded to d' when k does not divide d); m = d' / k; N = codebook size, a power of two
 * in [2, 65536]; B = log2 N; P = ceil(m * B / 8) = fq_payload_bytes(d, k, N).
 *
 * Record layout (a fixed-rate, fixed-address format, two planes):
 *   codes plane: n records of P bytes, record t at byte offset t * P.  Index j of a record
 *                occupies record bits [j*B, (j+1)*B), least significant bit first; record bit
 *                i is bit (i % 8) of byte (i / 8); unused tail bits are zero.
 *   norms plane: n IEEE fp16 values (passed as uint16_t bit patterns), norm t at element t.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers unless the comment says "host".  The caller owns
 *     every buffer; the library never allocates device memory and keeps no state between calls
 *     (fq_attn_decode_noalloc, below, is the one exception: it uses a fixed library array).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and is
 *     asynchronous; results are valid once the stream has reached the enqueued work.
 *   - Errors are returned as fq_status from host-side validation before anything is enqueued,
 *     or FQ_ERR_CUDA when a launch fails.  Nothing aborts or throws across the ABI.
 *   - n = 0 (or T = 0 in attention) is a valid no-op returning FQ_OK.
 *   - Limits: 1 <= d <= 256, 1 <= k <= d, N a power of two in [2, 65536]; other values
 *     return FQ_ERR_UNSUPPORTED.  Non-finite inputs are a precondition violation and
 *     are not detected.
 *   - Rotation `rot`: d' x d' fp32, row-major, z = rot * pad(x) (rows = output coordinates).
 *     Codebook `codebook`: N x k fp32, row-major.  Both are plain input data; the library
 *     reads them on every call (they are small: at most 256 KB and 2 MB).
 */
#ifndef FQ_H_
#define FQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FQ_OK = 0,
  FQ_ERR_INVALID_ARG = 1, /* null pointer for a non-empty call, negative size, bad enum */
  FQ_ERR_UNSUPPORTED = 2, /* a size outside the limits above */
  FQ_ERR_ALIGNMENT = 3,   /* a pointer that breaks a stated alignment rule */
  FQ_ERR_WORKSPACE = 4,   /* workspace / index buffer missing or too small */
  FQ_ERR_CUDA = 5,        /* a CUDA launch or runtime call failed */
  FQ_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (see fq_wait_status) */
} fq_status;

typedef enum { FQ_F16 = 0, FQ_F32 = 1 } fq_dtype;

/* Search-index kinds for fq_build_search_index. */
typedef enum {
  FQ_INDEX_EXACT = 0, /* conservative candidate lists: identical results to brute force */
  FQ_INDEX_TOPC = 1,  /* Cartesian grid, c codewords nearest each cell centre (approximate) */
  FQ_INDEX_TENSOR = 2 /* the codebook as tensor-core operand tiles, for half- and full-vector
                         codes (k = 32 or 64): brute-force GEMM search, brute-force results */
} fq_index_kind;

/* Decoder rescale rules (Block Sphere VQ notes, key design 3), for fq_decode_rescaled. */
typedef enum {
  FQ_RESCALE_PLAIN = 0,    /* S = 1: the plain decoder, as fq_decode */
  FQ_RESCALE_MSE = 1,      /* S = rho / |zbar|^2: least squared reconstruction error */
  FQ_RESCALE_UNBIASED = 2  /* S = 1 / rho: unbiased inner products */
} fq_rescale_rule;

/* ABI version of this header (bumped on any incompatible change). */
int fq_abi_version(void);

/* Static, NUL-terminated description of a status code. */
const char* fq_status_string(fq_status status);

/* d' = k * ceil(d / k), or 0 when (d, k) is unsupported. */
int fq_padded_dim(int d, int k);

/* P, the payload bytes of one record (summary sec. 2.3: b = log2(N)/k bits per coordinate,
 * so m * log2(N) bits per vector), or 0 when (d, k, N) is unsupported. */
size_t fq_payload_bytes(int d, int k, int N);

/*
 * fq_encode - the FibQuant encoder (summary sec. 2.3 "encoder").
 *   x          [n, d] row-major, fp16 or fp32 (x_type); any 2-byte (fp16) / 4-byte (fp32)
 *              aligned address.
 *   rot        [d', d'] fp32 Haar rotation.       codebook  [N, k] fp32.
 *   codes      [n, P] bytes (output), any address.  norms [n] fp16 bits (output), 2-byte aligned.
 *   search_index  NULL for brute force over all N codewords, or a device copy of a buffer
 *              made by fq_build_search_index for this exact codebook, d and k (8-byte aligned).
 * A zero vector encodes as norm +0 with all indices 0.  Ties between codewords resolve to
 * the lowest index.  FQ_INDEX_EXACT gives the brute-force result; FQ_INDEX_TOPC may not.
 */
fq_status fq_encode(const void* x, fq_dtype x_type, int64_t n, int d, int k, int N,
                    const float* rot, const float* codebook, uint8_t* codes, uint16_t* norms,
                    const void* search_index, void* stream);

/*
 * fq_decode - the FibQuant decoder (summary sec. 2.3 "decoder"): y_t = nu_t (Pi^T zhat_t)[0:d]
 * with zhat_t the concatenated codewords of record t.
 *   codes [n, P], norms [n] as produced by fq_encode (norms 2-byte aligned).
 *   y     [n, d] output, fp32 or fp16 (y_type, fp16 is round-to-nearest-even of the fp32
 *         result); 4-byte (fp32) or 2-byte (fp16) aligned.
 * Random access: to decode tokens [t0, t0 + n) pass codes + t0 * P and norms + t0.
 */
fq_status fq_decode(const uint8_t* codes, const uint16_t* norms, int64_t n, int d, int k, int N,
                    const float* rot, const float* codebook, void* y, fq_dtype y_type,
                    void* stream);

/*
 * fq_decode_gather - random access (summary sec. 1: every record sits at a fixed address, so
 * any token decodes alone): y[i] = decode of record token_ids[i], for a token list in any order
 * with repeats allowed.
 *   codes, norms   a plane of n_records records (as produced by fq_encode).
 *   token_ids      [n_ids] int64 device array, 8-byte aligned.  An id outside [0, n_records)
 *                  reads nothing and gives a row of NaN (ids live on the device, so they are
 *                  checked there, not on the host).
 *   y              [n_ids, d] output, fp32 or fp16 (y_type), aligned as in fq_decode.
 * Results equal fq_decode of the listed records.
 */
fq_status fq_decode_gather(const uint8_t* codes, const uint16_t* norms, int64_t n_records,
                           const int64_t* token_ids, int64_t n_ids, int d, int k, int N,
                           const float* rot, const float* codebook, void* y, fq_dtype y_type,
                           void* stream);

/*
 * fq_encode_rho - fq_encode that also stores, per vector, the alignment rho = <z, zbar> of the
 * unit rotated vector z with its reconstruction zbar (the concatenated codewords), the one extra
 * scalar of BlockQuant's target-aware rescale (Block Sphere VQ notes, key design 3).
 *   rho  [n] fp16 bits (output, 2-byte aligned), round to nearest even; 1 for a zero vector.
 * Everything else as fq_encode (same records and norms).  Runs the one-warp-per-vector kernel.
 */
fq_status fq_encode_rho(const void* x, fq_dtype x_type, int64_t n, int d, int k, int N,
                        const float* rot, const float* codebook, uint8_t* codes,
                        uint16_t* norms, uint16_t* rho, const void* search_index, void* stream);

/*
 * fq_decode_rescaled - the decoder with the rescale of Block Sphere VQ key design 3:
 *   y_t = nu_t S_t (Pi^T zbar_t)[0:d],  S_t from `rule` (fq_rescale_rule) and the stored rho_t:
 *   FQ_RESCALE_MSE S = rho / |zbar|^2, FQ_RESCALE_UNBIASED S = 1 / rho, FQ_RESCALE_PLAIN S = 1.
 *   rho  [n] fp16 bits as written by fq_encode_rho.  Everything else as fq_decode.
 */
fq_status fq_decode_rescaled(const uint8_t* codes, const uint16_t* norms, const uint16_t* rho,
                             int64_t n, int d, int k, int N, const float* rot,
                             const float* codebook, int rule, void* y, fq_dtype y_type,
                             void* stream);

/*
 * fq_encode_prod / fq_decode_prod - TurboQuant_prod (TurboQuant notes sec. 3.2), the unbiased
 * inner-product quantizer that FibQuant is compared with: a scalar (k = 1) MSE code of the
 * rotated unit vector at b - 1 bits per coordinate, plus the 1-bit QJL sketch (sec. 2.2) of its
 * residual and the residual's norm.
 *   encode: nu = |x|, u = x / nu, y = rot u, idx_r = nearest level of c1 to y_r (lowest index on
 *           ties), r = u - rot^T c1[idx], gamma = |r|, q = sign(qjl r) with sign(0) = +1.
 *   decode: y = nu (rot^T c1[idx] + gamma sqrt(pi/2) / d qjl^T q).
 *   N1        levels of the scalar codebook c1 ([N1] fp32, a power of two in [2, 256]).
 *   rot, qjl  [d, d] fp32: the Haar rotation and the QJL matrix (iid N(0,1) entries).
 *   codes     [n, P1] bytes, P1 = fq_payload_bytes(d, 1, N1): index r at bits [r B1, (r+1) B1).
 *   signs     [n, ceil(d / 8)] bytes: bit r % 8 of byte r / 8 is set when q_r = +1.
 *   norms, gamma  [n] fp16 bits each (round to nearest even).
 * Runs one warp per vector; d <= 256.
 */
fq_status fq_encode_prod(const void* x, fq_dtype x_type, int64_t n, int d, int N1,
                         const float* rot, const float* c1, const float* qjl, uint8_t* codes,
                         uint8_t* signs, uint16_t* norms, uint16_t* gamma, void* stream);
fq_status fq_decode_prod(const uint8_t* codes, const uint8_t* signs, const uint16_t* norms,
                         const uint16_t* gamma, int64_t n, int d, int N1, const float* rot,
                         const float* c1, const float* qjl, void* y, fq_dtype y_type,
                         void* stream);

/*
 * Workspace bytes fq_attn_decode needs for these sizes (the split-softmax partials), or 0
 * when the sizes are unsupported.  The value depends only on the arguments.
 */
size_t fq_attn_workspace_bytes(int B, int Hq, int Hkv, int64_t T, int d, int kV);

/*
 * fq_attn_decode - one decode-attention step over a FibQuant-compressed KV cache:
 *   out[b, h] = sum_t softmax_t(scale * q[b,h] . khat[b,g,t]) vhat[b,g,t],  g = h / (Hq/Hkv),
 * computed without decompressing: q is rotated once by Pi_K, scores come from per-block
 * dot-product tables LUT[j][c] = (Pi_K q)_j . C_K[c] times the key norm, values are
 * accumulated in the rotated domain and rotated back by Pi_V^T once per head.
 *   q        [B, Hq, d] fp16 bits.         out [B, Hq, d] fp32.
 *   k_codes  [B, Hkv, T, P_K] bytes;  k_norms [B, Hkv, T] fp16 bits (kK, NK, rotK, cbK).
 *   v_codes  [B, Hkv, T, P_V] bytes;  v_norms [B, Hkv, T] fp16 bits (kV, NV, rotV, cbV).
 *   workspace  device buffer of at least fq_attn_workspace_bytes(...) bytes, 16-byte aligned,
 *              owned by the caller, overwritten by the call (no state survives it).
 * Requires Hkv >= 1, Hq % Hkv == 0, Hq / Hkv <= 16, T >= 1, d <= 128, N_K, N_V <= 1024.
 */
fq_status fq_attn_decode(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                         const uint8_t* k_codes, const uint16_t* k_norms, int kK, int NK,
                         const float* rotK, const float* cbK,
                         const uint8_t* v_codes, const uint16_t* v_norms, int kV, int NV,
                         const float* rotV, const float* cbV,
                         float scale, float* out, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * fq_attn_decode_lengths - fq_attn_decode over caches of capacity T whose sequences have their
 * own context lengths (summary sec. 1: a sequence may end anywhere; records past its end are
 * never read and may hold anything).
 *   lengths  [B] int32 device array, 4-byte aligned: sequence b attends over its first
 *            clamp(lengths[b], 0, T) tokens; a sequence of length 0 outputs zeros.
 *   Everything else as fq_attn_decode (layouts [B, Hkv, T, P]; workspace of
 *   fq_attn_workspace_bytes(B, Hq, Hkv, T, d, kV) bytes).
 */
fq_status fq_attn_decode_lengths(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                                 const int32_t* lengths, const uint8_t* k_codes,
                                 const uint16_t* k_norms, int kK, int NK, const float* rotK,
                                 const float* cbK, const uint8_t* v_codes,
                                 const uint16_t* v_norms, int kV, int NV, const float* rotV,
                                 const float* cbV, float scale, float* out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * fq_attn_decode_append - one decode step that writes its own token: the write path of the
 * cache fused into the attention step.
 *   k_new, v_new  [B, Hkv, d] fp16 bits: the step's key and value.  Each is encoded (brute-force
 *                 search, as fq_encode) into record slot lengths[b] of its sequence in
 *                 k_codes/k_norms and v_codes/v_norms ([B, Hkv, T, P] planes, written in place).
 *   lengths       [B] int32 device array, in/out: tokens already in each sequence.  The step
 *                 attends over lengths[b] + 1 tokens (the cache plus the new token) and, when it
 *                 completes, adds one to lengths[b].  A sequence already holding T tokens is
 *                 not written and not advanced (it attends over its T tokens).
 *   Everything else as fq_attn_decode.  T must be at least 1.
 * Enqueued as: encode of the new keys, encode of the new values, attention, combine (which
 * advances lengths after every read of it).
 */
fq_status fq_attn_decode_append(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                int B, int Hq, int Hkv, int64_t T, int d, int32_t* lengths,
                                uint8_t* k_codes, uint16_t* k_norms, int kK, int NK,
                                const float* rotK, const float* cbK, uint8_t* v_codes,
                                uint16_t* v_norms, int kV, int NV, const float* rotV,
                                const float* cbV, float scale, float* out, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Size of the fixed device scratch used by fq_attn_decode_noalloc (4 MiB per GPU). */
#define FQ_ATTN_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * fq_attn_decode_noalloc - fq_attn_decode for callers that cannot allocate device memory.
 * (No counterpart in the paper: this is a convenience of this library.)
 *
 * fq_attn_decode needs a caller-owned workspace for its split-softmax partials.  Callers that
 * cannot allocate one - code running inside a host application whose allocator owns all
 * device memory, or a decode loop that must not call cudaMalloc because allocation may
 * synchronise the device and has unbounded latency - can call this instead.  It keeps the
 * partials in a fixed array of FQ_ATTN_NOALLOC_SCRATCH_BYTES that every GPU loading this
 * library holds until the process exits, and it allocates nothing.
 *   Arguments, layouts, limits and results are those of fq_attn_decode without the workspace.
 *   Sizes whose fq_attn_workspace_bytes(...) exceeds FQ_ATTN_NOALLOC_SCRATCH_BYTES return
 *   FQ_ERR_WORKSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress
 *   with that device current); make that first call before any stream capture.
 *   All calls on a device share the one array: calls that overlap on the GPU (for example on
 *   two streams at once) race and give undefined results; calls ordered on one stream are
 *   safe.  Nothing in the array needs to start at zero (every partial read is written first
 *   by the same call).
 */
fq_status fq_attn_decode_noalloc(const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d,
                                 const uint8_t* k_codes, const uint16_t* k_norms, int kK,
                                 int NK, const float* rotK, const float* cbK,
                                 const uint8_t* v_codes, const uint16_t* v_norms, int kV,
                                 int NV, const float* rotV, const float* cbV, float scale,
                                 float* out, void* stream);

/*
 * fq_wait_status - reports kernels whose bounded device-side waits gave up.
 *
 * Every wait inside the library's kernels (for an asynchronous copy, a tensor-core operation or
 * another warp's hand-off) gives up after a bounded number of polls instead of hanging the GPU.
 * A CTA whose wait gave up stops its loop, lets its own copies and tensor-core work in flight
 * land, frees its tensor memory, adds one to a per-GPU failure count and exits; the outputs of
 * that launch are then unspecified.  Launches are asynchronous, so the entry points above cannot
 * return FQ_ERR_TIMEOUT themselves; this call reports it.
 *   timed_out  (host, out, may be NULL) the number of CTAs whose waits gave up on the current
 *              device since the count was last cleared.
 *   clear      nonzero: reset the count to zero after reading it.
 * Waits for all work on the current device first (cudaDeviceSynchronize), so do not call it
 * inside a stream capture.  Returns FQ_ERR_TIMEOUT when the count is nonzero, FQ_OK when it is
 * zero, FQ_ERR_CUDA when the device cannot be queried.
 */
fq_status fq_wait_status(unsigned* timed_out, int clear);

/*
 * fq_selftest_wait_timeout - diagnostic for the failure path (no counterpart in the paper).
 * Enqueues on `stream` one small kernel whose single wait is on an mbarrier phase that nothing
 * ever completes; it polls `polls` times (1 .. 2^20), gives up exactly as the codec kernels do
 * and counts one timed-out wait, which fq_wait_status then reports.  Nothing faults or hangs.
 */
fq_status fq_selftest_wait_timeout(uint32_t polls, void* stream);

/*
 * fq_build_search_index - builds, on the HOST, the candidate table fq_encode can use instead
 * of brute force (Block Sphere VQ notes, key design 2, "Cartesian LUT": a grid of L cells per
 * axis over the block space, each cell holding a short candidate list).
 *   codebook_host  [N, k] fp32 host array (the same values later passed to fq_encode).
 *   d              vector length the index will be used with (sets the grid range).
 *   kind           FQ_INDEX_EXACT: every codeword that can be nearest to some point of the
 *                  cell is listed (so the search equals brute force); c is ignored.
 *                  FQ_INDEX_TOPC: the c codewords nearest to each cell centre (approximate).
 *                  FQ_INDEX_TENSOR: no grid (L and c are ignored); the codebook laid out as
 *                  tensor-core operand tiles for half- and full-vector codes (k a multiple of
 *                  16, at most 64; N at least 256 for k <= 32, 128 otherwise).  fq_encode then
 *                  searches all N codewords on the tensor cores (d = 64 with k = 32 or 64,
 *                  d = 128 with k = 64; other shapes ignore it) and returns the brute-force
 *                  result (up to near ties of ~2^-20).  The device copy must be 16-byte aligned.
 *   L              cells per axis (2..256; L^k <= 2^22).
 *   index_host     host output buffer of index_capacity bytes, or NULL to query the size.
 *   index_bytes    (host, out) the exact size the index needs.
 * Returns FQ_ERR_WORKSPACE (with *index_bytes set) when index_host is NULL or too small.
 * The caller copies the buffer to device memory (8-byte aligned) and passes it to fq_encode.
 */
fq_status fq_build_search_index(const float* codebook_host, int d, int k, int N, int kind,
                                int L, int c, void* index_host, size_t index_capacity,
                                size_t* index_bytes);

#ifdef __cplusplus
}
#endif

#endif /* FQ_H_ */
