/*
 * magicpig.h - C ABI of the B200 (sm_100a) LSH-sampled decode-attention library.
 *
 * Method: MagicPIG, "LSH Sampling for Efficient LLM Generation" (Chen et al.,
 * 2024).  The GrooveSquid summary page ("Medium Difficulty Summary") describes
 * it as estimating the attention output by sampling instead of TopK selection;
 * the sourcepulse project page ("How It Works") says the samples are chosen by
 * locality-sensitive hashing; the gitdiagram page ("LSH Sampling": LSH kernel,
 * LSH interface) names a native LSH library under it.  The arithmetic, in the
 * notation used throughout this library:
 *
 *   SimHash.  W holds L*K random hyperplanes of dimension d; row c = l*K + b is
 *   the hyperplane of bit b of table l.  Bit b of the table-l code of a vector
 *   x is 1 iff x . W[c] > 0 (exactly 0 gives 0).
 *   Sampling.  A context token i outside the exact set D is sampled for query
 *   head h (i in S_h) iff its code equals the query's in at least 2 of the L
 *   tables.  D = [0, sink) U [N - window, N).
 *   Estimator.  s_i = q . k_i / sqrt(d); p_i = 1 - arccos(cos(q, k_i)) / pi;
 *   x_i = p_i^K; u_i = 1 - (1-x_i)^L - L x_i (1-x_i)^(L-1); w_i = exp(s_i) on
 *   D and exp(s_i - log u_i) on S_h; out = sum w_i v_i / sum w_i over D U S_h;
 *   lse = log sum w_i (natural log, -log u included).
 *
 * Conventions for every call:
 *   - Tensors are caller-owned device buffers (bf16 is passed as raw 16-bit
 *     patterns).  The library allocates nothing.  Its global state is a
 *     per-device cache of function attributes and, for
 *     mp_decode_attend_noalloc only, one fixed 16 MiB scratch array in device
 *     memory on every GPU that loads the library (with its address cached per
 *     device).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) except mp_read_status, which synchronises.
 *   - Return value: MP_OK or a negative MP_ERR_* from host-side validation
 *     (nothing is launched then) or from the CUDA launch itself.  Faults found
 *     on the device (a sequence length past the capacity) never trap: they are
 *     written to a status word and the offending length is clamped.
 *   - Every device pointer must be 16-byte aligned.
 */
#ifndef MAGICPIG_H
#define MAGICPIG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MP_OK 0
#define MP_ERR_ARG (-1)       /* null pointer, negative size, bad value */
#define MP_ERR_SHAPE (-2)     /* unsupported shape (see mp_shape) */
#define MP_ERR_ALIGN (-3)     /* a pointer is not 16-byte aligned */
#define MP_ERR_CAPACITY (-4)  /* a length exceeds the capacity / max_len (device: clamped) */
#define MP_ERR_WORKSPACE (-5) /* workspace smaller than mp_decode_workspace_bytes */
#define MP_ERR_CUDA (-6)      /* a CUDA runtime call or launch failed */
#define MP_ERR_TOO_LARGE (-7) /* beyond the fixed scratch of mp_decode_attend_noalloc */

/* Key-code layouts (mp_shape.code_layout). */
#define MP_CODES_AUTO 0   /* MP_CODES_PLANES, except MP_CODES_BYTES for k_bits == 8 when
                             batch * n_kv_heads * capacity < MP_CODES_AUTO_PLANES_MIN */
#define MP_CODES_BYTES 1  /* one byte per (table, token); k_bits == 8 only */
#define MP_CODES_PLANES 2 /* bit planes of 32 tokens; any supported k_bits */
/* Below this many (token, kv head) slots a K = 8 scan has too few 1024-token
   chunks to fill the GPU with one warp each, and byte codes (512-token chunks)
   scan faster: measured on one B200, 1 x 8 x 16.5k slots decode in 34 us with
   bytes against 40 us with planes, 4 x 8 x 131k slots in 116 us with planes
   against 118 us with bytes, 16 x 8 x 131k in 383 against 411 us. */
#define MP_CODES_AUTO_PLANES_MIN (1 << 21)

/*
 * Problem shape.  Supported: head_dim == 128; k_bits in {8, 10};
 * 2 <= n_tables <= 255 with n_tables * k_bits <= 2048; n_q_heads a multiple of
 * n_kv_heads with group G = n_q_heads / n_kv_heads in {1, 2, 4, 8};
 * capacity a positive multiple of 128 below 2^24; sink, window >= 0.
 */
typedef struct mp_shape {
    int32_t batch;      /* B */
    int32_t n_q_heads;  /* Hq */
    int32_t n_kv_heads; /* Hkv */
    int32_t head_dim;   /* d */
    int32_t capacity;   /* Ncap: token slots of the K/V caches and of the codes */
    int32_t k_bits;     /* K: SimHash bits per table */
    int32_t n_tables;   /* L: hash tables */
    int32_t sink;       /* leading tokens of the exact set D */
    int32_t window;     /* trailing (most recent) tokens of the exact set D */
    int32_t code_layout; /* MP_CODES_AUTO, MP_CODES_BYTES or MP_CODES_PLANES */
} mp_shape;

/*
 * Key-code layouts ("table-major"), per (b, kv head) unit:
 *   MP_CODES_BYTES  (k_bits == 8): uint8 [B][Hkv][L][Ncap], one byte per
 *                   (table, token), bit b of the byte = bit b of the code.
 *   MP_CODES_PLANES: uint32 [B][Hkv][L][Ncap/32][K] bit planes: bit t of word
 *                   (l, w, b) = bit b of the table-l code of token 32*w + t
 *                   (the K planes of each 32-token group are adjacent).
 * Both use exactly L*K/8 bytes per token; mp_codes_bytes gives the size.  The
 * plane layout lets the collision scan test 32 tokens per logical operation
 * (K + 2 operations per 32 tokens and query head, against one packed compare
 * per token and head for bytes), which MP_CODES_AUTO uses except on small
 * K = 8 problems.
 */
int mp_codes_bytes(const mp_shape *shape, size_t *bytes);

/*
 * Key hashing (SimHash of cached keys; the "LSH kernel" / hash-table
 * construction of the gitdiagram and sourcepulse pages).
 *   keys   bf16 [B][Hkv][Ncap][d]   rows [0, n_tokens) of every unit are hashed
 *   W      bf16 [L*K][d]            hyperplanes, row c = l*K + b
 *   seq_lens  int32 [B] device, nullable: if given, unit (b, .) hashes only
 *          tokens [0, min(seq_lens[b], n_tokens)) (ragged batches)
 *   codes  out, layout above; only the hashed tokens are written (with bit
 *          planes the last partial 32-token word is rewritten whole).
 *   status int32 device word (nullable): MP_ERR_CUDA if the kernel's internal
 *          pipeline stalled (a bounded wait expired; the codes are then
 *          incomplete).  Never written on success.
 * 0 <= n_tokens <= Ncap (host bound; sizes the grid).  Projections are bf16
 * tensor-core products with fp32 accumulation (tcgen05).
 */
int mp_hash_keys(const mp_shape *shape, const void *keys, const void *W, const int32_t *seq_lens,
                 int32_t n_tokens, void *codes, int32_t *status, void *stream);

/*
 * Streamed key hashing: SimHash of the token range [first_token, first_token +
 * n_tokens) of every (b, kv head) unit, for a prefill that fills the cache
 * block by block (the pages' "optimized hash table construction", done while
 * the cache grows).  Same kernel and arithmetic as mp_hash_keys; nothing
 * outside the range is read, and for the byte layout nothing outside it is
 * written.  It can run on a second stream next to mp_decode_attend calls that
 * read only tokens below first_token.
 *   first_token  multiple of 128 (the kernel's row tile); else MP_ERR_ALIGN
 *   n_tokens     >= 0, first_token + n_tokens <= Ncap (else MP_ERR_CAPACITY)
 *   keys, W, codes, status, stream as for mp_hash_keys.  With bit-plane codes
 *   the 32-token word holding the range's last token is written whole: its
 *   bits for tokens past the range are cleared (they are hashed with a later
 *   block).
 */
int mp_hash_keys_range(const mp_shape *shape, const void *keys, const void *W, int32_t first_token,
                       int32_t n_tokens, void *codes, int32_t *status, void *stream);

/*
 * Query hashing: qcodes[b][h][l] (uint16) = table-l SimHash code of q[b][h].
 *   q bf16 [B][Hq][d]; W as above; qcodes out uint16 [B][Hq][L].
 */
int mp_hash_queries(const mp_shape *shape, const void *q, const void *W, uint16_t *qcodes,
                    void *stream);

/*
 * Decode-time append of one token per sequence: for every (b, kv head), at
 * pos = seq_lens[b], writes k_cache/v_cache rows from k_new/v_new, writes the
 * SimHash codes of k_new into column pos of the codes, then seq_lens[b] += 1.
 *   k_new, v_new  bf16 [B][Hkv][d]
 *   k_cache, v_cache  bf16 [B][Hkv][Ncap][d]      codes  layout above
 *   seq_lens  int32 [B] device, incremented in place
 *   status    int32 device word (nullable): set to MP_ERR_CAPACITY when some
 *             seq_lens[b] >= Ncap (that sequence is then left untouched).
 */
int mp_append_token(const mp_shape *shape, const void *k_new, const void *v_new, const void *W,
                    void *k_cache, void *v_cache, void *codes, int32_t *seq_lens,
                    int32_t *status, void *stream);

/* Kernel paths of mp_decode_attend (mp_decode_debug.path). */
#define MP_PATH_AUTO 0     /* the faster path for the shape: currently always MP_PATH_SPLIT */
#define MP_PATH_SPLIT 1    /* collision scan, then sampled attention (two kernels) */
#define MP_PATH_FUSED 2    /* one kernel scans and attends (bit-plane codes, G <= 4);
                              MP_ERR_SHAPE where it does not apply */
#define MP_PATH_TC 3       /* collision scan, then sampled attention on the tcgen05 tensor cores
                              (scores, key norms and P.V in TMEM; persistent, one CTA per SM) */

/* Test hooks of mp_decode_attend (all nullable / zero). */
typedef struct mp_decode_debug {
    const uint16_t *qcodes_in; /* [B][Hq][L]: use these query codes instead of hashing q */
    uint16_t *qcodes_out;      /* [B][Hq][L]: copy of the query codes used */
    uint8_t *member_out;       /* [B][Hq][Ncap]: 1 iff token i is in S_h (i < N_b) */
    int32_t path;              /* MP_PATH_*: which kernel path to take */
    int32_t skip_scan;         /* nonzero: launch no collision scan (MP_PATH_AUTO / MP_PATH_SPLIT
                                  only, else MP_ERR_ARG), so that the attention's bounded waits for
                                  the scan's per-chunk ready flags run out: each waiting block gives
                                  up after 1 s, records MP_ERR_CUDA in the status word and returns
                                  without reading a candidate list; out / lse / n_sampled are then
                                  undefined.  Tests the failure path without a GPU fault. */
} mp_decode_debug;

/* Workspace bytes that mp_decode_attend needs for sequences up to max_len. */
int mp_decode_workspace_bytes(const mp_shape *shape, int32_t max_len, size_t *bytes);

/*
 * One LSH-sampled decode step (query hashing, collision scan + compaction,
 * sampled attention with the -log u correction, the exact sink/window set D
 * and the log-sum-exp merge) for every (b, query head).
 *   q        bf16 [B][Hq][d]          W bf16 [L*K][d]
 *   codes    key codes (layout above), valid for tokens [0, seq_lens[b])
 *   k_cache, v_cache  bf16 [B][Hkv][Ncap][d]
 *   seq_lens int32 [B] device: N_b; each must be <= max_len (else clamped and
 *            MP_ERR_CAPACITY is recorded in the status word)
 *   max_len  host bound on every N_b, 0 <= max_len <= Ncap (sizes the grid)
 *   out      fp32 [B][Hq][d]           lse fp32 [B][Hq] (-inf when N_b == 0)
 *   n_sampled int32 [B][Hq]: |S_h|, tokens of D excluded
 *   workspace device scratch of at least mp_decode_workspace_bytes bytes; its
 *            first word is the status word (reset by every call)
 *   debug    nullable test hooks
 */
int mp_decode_attend(const mp_shape *shape, const void *q, const void *W, const void *codes,
                     const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                     int32_t max_len, float *out, float *lse, int32_t *n_sampled, void *workspace,
                     size_t workspace_bytes, const mp_decode_debug *debug, void *stream);

/*
 * mp_decode_attend without a caller-provided workspace.  The method has no
 * counterpart of this call: it exists for callers that cannot allocate device
 * memory where they decode — runtimes whose memory pools are sealed after
 * start-up, plugins that only receive tensors from a host framework and may
 * not call cudaMalloc themselves.  Same arguments, results and device checks
 * as mp_decode_attend, minus the workspace and the test hooks.
 *   - Scratch is one fixed array of 16 MiB compiled into the library; every
 *     GPU that loads the library holds it until the process exits.
 *   - Problems whose workspace (mp_decode_workspace_bytes) exceeds 16 MiB are
 *     rejected with MP_ERR_TOO_LARGE before anything is launched (a single
 *     128k-token sequence with 8 kv heads and K = 8 fits).
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it: make that first call before any
 *     stream capture begins.  The cached address belongs to the device's
 *     current context: after a device reset (cudaDeviceReset) it is stale, and
 *     the library must be unloaded and loaded again before this call is used
 *     on that device.
 *   - Every call shares the array: calls whose executions overlap on the GPU
 *     (several streams or host threads on one device) race and must be
 *     serialised by the caller.  The array's contents carry over between calls;
 *     nothing in it needs to start at zero.
 *   - status: int32 device word (nullable) that receives this call's status
 *     word (MP_OK or MP_ERR_CAPACITY), copied asynchronously on `stream`.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
int mp_decode_attend_noalloc(const mp_shape *shape, const void *q, const void *W, const void *codes,
                             const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                             int32_t max_len, float *out, float *lse, int32_t *n_sampled,
                             int32_t *status, void *stream);

/*
 * int8 keys for the attention gather (opt-in; the method itself reads the
 * cached keys in their own precision, so this is a reduced-precision variant
 * of the step, not part of the method's description).  The bf16 key cache
 * stays authoritative for hashing: the codes are always computed from bf16
 * keys, and the int8 copy only replaces the K rows that the sampled attention
 * gathers (144 bytes per row instead of 256; the V rows and codes are
 * unchanged).
 *
 * Format: row (b, h, i) of the bf16 keys k (d = 128 values) is stored as 144
 * contiguous bytes, k8[b][h][i][0 .. 143]:
 *   bytes 0 .. 127    q_j = rint(k_j / s)   (round half to even; int8 in [-127, 127])
 *   bytes 128 .. 143  the record {s, |s q|^2, 0, 0}   (fp32 x 4)
 * where s = 2^e is the smallest power of two with 127 s >= max_j |k_j| (s = 0
 * and q = 0 for a zero row).  s is a power of two, so s * q is exactly a bf16
 * value and the stored squared norm is exact: the attention runs on the keys
 * k~ = s * q, |k_j - k~_j| <= s/2 <= max|k| / 127, and an exact bf16 cache of
 * k~ gives the same result through mp_decode_attend.  Queries enter the
 * score products as f16 (exact for bf16 values of magnitude 2^-17 .. 65504).
 * Expected cost, measured on the fp64 estimator: about 1e-2 relative L2 on
 * the output of a head.
 *   k8  int8 [B][Hkv][Ncap][MP_Q8_ROW_BYTES], 16-byte aligned, caller-owned
 */
#define MP_Q8_ROW_BYTES 144

/*
 * Writes the int8 rows (k8) of key rows [first_token, first_token +
 * n_tokens) of every (b, kv head), stopping at seq_lens[b] when seq_lens
 * (int32 [B], device, nullable) is given.  Errors: MP_ERR_ARG (null pointer),
 * MP_ERR_ALIGN, MP_ERR_CAPACITY (range outside [0, Ncap]); nothing launched.
 */
int mp_quantize_keys(const mp_shape *shape, const void *k_cache, const int32_t *seq_lens, int32_t first_token,
                     int32_t n_tokens, int8_t *k8, void *stream);

/*
 * mp_append_token that also writes the int8 row of each appended key into
 * k8 at the same position (one launch).  Same arguments and status behaviour
 * as mp_append_token otherwise, except that k_cache may be NULL: then no bf16
 * key row is written, and a caller that decodes only through
 * mp_decode_attend_q8 keeps 400 instead of 512 bytes of key-value cache per
 * (token, kv head) (the bf16 keys are needed again only to rebuild the codes,
 * e.g. for a new W).
 */
int mp_append_token_q8(const mp_shape *shape, const void *k_new, const void *v_new, const void *W,
                       void *k_cache, void *v_cache, void *codes, int32_t *seq_lens, int8_t *k8, int32_t *status,
                       void *stream);

/*
 * mp_decode_attend with the K rows gathered from the int8 rows (k8) instead
 * of a bf16 cache; every other argument and result as there.
 * debug->path may be MP_PATH_AUTO or MP_PATH_SPLIT; MP_PATH_FUSED and
 * MP_PATH_TC return MP_ERR_SHAPE (those kernels read bf16 keys only).
 */
int mp_decode_attend_q8(const mp_shape *shape, const void *q, const void *W, const void *codes,
                        const int8_t *k8, const void *v_cache, const int32_t *seq_lens, int32_t max_len,
                        float *out, float *lse, int32_t *n_sampled, void *workspace, size_t workspace_bytes,
                        const mp_decode_debug *debug, void *stream);

/* Synchronises `stream` and reads the status word of a decode workspace. */
int mp_read_status(const void *workspace, int32_t *status, void *stream);

/* Human-readable name of an MP_* code. */
const char *mp_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* MAGICPIG_H */
