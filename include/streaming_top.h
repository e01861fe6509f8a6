/*
 * streaming_top -- C ABI of the B200 (sm_100a) CSA lightning-indexer top-k.
 *
 * The operation (StreamIndex, "Memory-Bounded Compressed Sparse Attention via
 * Streaming Top-k", abstract: the lightning indexer scores the compressed keys
 * and the top-k are selected per query, by a chunked partition-merge top-k that
 * never materialises the [B, S, H_I, T] fp32 score tensor).  The scoring
 * function is the DeepSeek-V3.2 lightning-indexer form (the lineage the
 * DeepSeek-V4.1 sparse-attention page gives the indexer, section "indexer"):
 *
 *     I[b,t,s] = sum_{h < H_I} w[b,t,h] * ReLU( sum_{d < D} q[b,t,h,d] * kc[b,s,d] )
 *
 * Compressed key s covers tokens [s*m, s*m+m-1] and is visible to query t iff
 * s*m+m-1 <= t and s < T.  For every (b, t) the result is the visible keys
 * with the k largest scores, sorted by score descending with the lower index
 * winning ties; when fewer than k keys are visible the tail is index -1 and
 * score -inf.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, dense
 *     row-major (C order), 16-byte aligned.  The library never frees or keeps
 *     them after the call returns.
 *   - Calls are asynchronous: they validate arguments on the host, enqueue
 *     work on `stream` (a cudaStream_t; NULL means the legacy default stream)
 *     and return.  A validation failure returns a status synchronously and
 *     enqueues nothing.  Device-side failures (a bounded wait that ran out) are
 *     reported by si_device_status().
 *   - The message of the last failure on the calling host thread is available
 *     from si_last_error().
 *   - Scratch a call needs and the caller does not pass (si_options.workspace)
 *     is allocated and freed on `stream` from a stream-ordered memory pool the
 *     library keeps per device; the pool holds up to 1 GiB of freed memory
 *     between calls so that repeated calls do not map memory anew.
 */
#ifndef STREAMING_TOP_H
#define STREAMING_TOP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SI_API __attribute__((visibility("default")))
#else
#define SI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum si_status {
  SI_OK = 0,
  SI_ERR_INVALID_ARGUMENT = 1, /* null pointer, non-positive size, misaligned pointer */
  SI_ERR_UNSUPPORTED = 2,      /* valid but outside what the kernels implement (D, H_I, k, key tile) */
  SI_ERR_OUT_OF_MEMORY = 3,    /* the path's memory need exceeds free device memory */
  SI_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed; see si_last_error() */
  SI_ERR_TIMEOUT = 5           /* a kernel's bounded wait ran out; the kernel exited early */
} si_status;

typedef enum si_dtype {
  SI_DTYPE_BF16 = 0,      /* q, kc are bf16 */
  SI_DTYPE_FP8_E4M3 = 1,  /* q, kc are OCP fp8 e4m3 codes with per-row fp32 scales */
  SI_DTYPE_MXFP4_KEYS = 2 /* q is bf16; kc is MXFP4 (the 4-bit indexer keys of the V4.1-Flash
                             deployment notes, "two-level sparse attention"): OCP Microscaling
                             FP4, E2M1 codes [B,T,D/2] bytes -- value d in the low nibble of byte
                             d/2 when d is even, the high nibble when odd -- with one E8M0 scale
                             per 32 values along D in kc_mx_scale [B,T,D/32] */
} si_dtype;

/* Options of si_indexer_topk_ex.  Zero-initialise, then set what you need. */
typedef struct si_options {
  si_dtype dtype;        /* SI_DTYPE_BF16 (default) or SI_DTYPE_FP8_E4M3 */
  const float* q_scale;  /* fp8 only: [B,S,H_I] fp32 > 0, value = code * scale (device) */
  const float* kc_scale; /* fp8 only: [B,T] fp32 > 0 (device) */
  int query_chunk;       /* queries per launch of the chunk driver; 0 = all S in one launch.
                            Must be a multiple of 4 otherwise. */
  int key_tile;          /* keys per partition of the partition-merge: 64 or a multiple
                            of 128 up to 1024; 0 = 512, or 256 / 128 / 64 when k is too
                            large for a 512-key partition's pool in shared memory.  An
                            explicit value whose pool does not fit gives SI_ERR_UNSUPPORTED. */
  void* workspace;       /* optional caller-owned device scratch, >= si_indexer_workspace_size() */
  size_t workspace_bytes;
  int unsorted;          /* streaming path only: 1 = leave each row's k results in an unspecified
                            order (valid entries first, then the -1 / -inf padding) and skip the
                            row sort; 0 (default) = sorted by score descending, index ascending */
  const uint8_t* kc_mx_scale; /* SI_DTYPE_MXFP4_KEYS only: E8M0 block scales [B,T,D/32], value
                            2^(byte-127) (device).  The keys are decoded to bf16 (exact for scales
                            <= 252) into B*T*D*2 bytes of scratch -- opt->workspace when given,
                            else allocated and freed on `stream` -- then scored as bf16. */
  int32_t* device_status;  /* optional: this call's own device error word, int32_t[2] in device
                            memory, 8-byte aligned, zeroed by the caller.  A kernel of the call
                            whose bounded wait runs out writes SI_ERR_TIMEOUT into [0] and the
                            waiting site into [1] (the first failure wins) and exits early.  NULL
                            (default): the library's per-device record, which si_device_status()
                            reads and clears, is used instead. */
} si_options;

/*
 * Streaming indexer top-k (the hot path).  Never allocates the
 * [B,S,H_I,T] score tensor.
 *   q       [B, S, H_I, D] bf16     kc [B, T, D] bf16     w [B, S, H_I] fp32
 *   out_idx [B, S, k] int32 (device, written)
 *   out_score [B, S, k] fp32 (device, written; may be NULL)
 * Supported: D == 128, H_I == 64, 1 <= k <= 2048, m >= 1, B, S, T >= 1.
 * Other shapes return SI_ERR_UNSUPPORTED.
 */
SI_API si_status si_indexer_topk(const void* q, const void* kc, const float* w, int B, int S, int T,
                          int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                          void* stream);

/* As si_indexer_topk, with options (dtype, fp8 scales, query chunk, key tile,
 * workspace).  opt may be NULL (defaults). */
SI_API si_status si_indexer_topk_ex(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                             void* stream, const si_options* opt);

/*
 * Streaming indexer top-k over a range of query rows: rows row0 .. row0+R-1
 * of every sequence, given as q [B, R, H_I, D] and w [B, R, H_I] (and for
 * fp8, q_scale [B, R, H_I]), against all T compressed keys kc [B, T, D];
 * results out_idx / out_score [B, R, k].  Row r is query position row0 + r
 * for causal visibility: key s is visible iff s*m + m - 1 <= row0 + r.  A
 * caller can so feed a long sequence's queries in chunks and hold only one
 * chunk of q on the device (the pages' streaming of the query side); each
 * row's result equals that of the whole-sequence call.  row0 >= 0, R >= 1,
 * row0 + R < 2^31; everything else as si_indexer_topk_ex.  No counterpart
 * of its own on the pages beyond that chunking of the queries.
 */
SI_API si_status si_indexer_topk_rows(const void* q, const void* kc, const float* w, int B, int row0,
                                      int R, int T, int H_I, int D, int m, int k, int32_t* out_idx,
                                      float* out_score, void* stream, const si_options* opt);

/*
 * Streaming indexer top-k on HOST buffers, end to end: rows row0 .. row0+R-1
 * of every sequence, laid out as si_indexer_topk_rows's arguments but in
 * host memory: q [B,R,H_I,D], w [B,R,H_I], kc [B,T,D] (all T keys), results
 * out_idx / out_score [B,R,k] (out_score may be NULL); for fp8, opt->q_scale
 * [B,R,H_I] and opt->kc_scale [B,T] are host pointers too, and for MXFP4
 * keys opt->kc_mx_scale [B,T,D/32].  row0 = 0, R = S is the whole sequence.
 * The pages stream the queries in chunks so that only one chunk is resident
 * (StreamIndex abstract, the memory bound at a million tokens); this call
 * does so from host memory: the keys are copied once, then chunks of
 * opt->query_chunk rows (0 = 4096; a multiple of 4) go through two device
 * slots, the copy of the next chunk in and of the previous chunk's results
 * out overlapping the scoring of the current one (two internal copy streams
 * ordered against `stream` by events).  Device memory: the keys plus two
 * chunks of q, w and results, si_indexer_topk_host_workspace_size() bytes,
 * from opt->workspace when given, else allocated and freed on `stream`.
 * Host buffers must stay valid for the call; page-locked memory
 * (cudaHostAlloc / cudaHostRegister) is needed for the copies to overlap,
 * pageable memory works but copies synchronously.  Blocks until the results
 * are in the host buffers.  Returns what si_indexer_topk_rows would, or
 * SI_ERR_TIMEOUT when a kernel's bounded wait ran out (read from
 * opt->device_status when given, else from the device record as
 * si_device_status() does).
 */
SI_API si_status si_indexer_topk_host(const void* q, const void* kc, const float* w, int B, int row0, int R,
                                      int T, int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                                      void* stream, const si_options* opt);

/* Device bytes si_indexer_topk_host needs for these arguments (its
 * opt->query_chunk and dtype; with_score != 0 when out_score is given). */
SI_API size_t si_indexer_topk_host_workspace_size(int B, int R, int T, int H_I, int D, int k, int with_score,
                                                  const si_options* opt);

/*
 * Sorts every row of a top-k result in place by (score descending, index
 * ascending): idx [rows, k] int32, score [rows, k] fp32, device memory, one
 * row per query.  Entries with index -1 and score -inf (padding) end up last.
 * This is the step si_indexer_topk runs after the streaming kernel when
 * out_score is given; callers that ran si_indexer_topk_ex with `unsorted`
 * can run it later.  Scores must not be NaN.  rows >= 0, 1 <= k <= 2048;
 * idx and score 4-byte aligned.  Asynchronous on `stream`.
 */
SI_API si_status si_sort_topk_rows(int32_t* idx, float* score, int64_t rows, int k, void* stream);

/*
 * Materialize path (in-library ground truth for small S, the method the
 * pages contrast with): writes the full [B,S,H_I,T] fp32 logits, reduces them
 * to [B,S,T] scores, then fully sorts every row.  Same arguments and results
 * as si_indexer_topk; any D >= 1 and H_I >= 1; T <= 16384.  Needs
 * 4*B*S*T*(H_I+1) bytes of scratch (taken from opt->workspace when given,
 * else allocated on `stream`); returns SI_ERR_OUT_OF_MEMORY without
 * allocating when that exceeds the free device memory.
 */
SI_API si_status si_indexer_materialize(const void* q, const void* kc, const float* w, int B, int S,
                                 int T, int H_I, int D, int m, int k, int32_t* out_idx,
                                 float* out_score, void* stream, const si_options* opt);

/*
 * Allocation-free variant of si_indexer_materialize, for callers that cannot
 * allocate device memory at call time (an application that has given nearly
 * all GPU memory to its own pool, a plugin step that must not allocate, a
 * latency-critical loop where cudaMalloc/cudaFree would synchronise).  It has
 * no counterpart on the pages: it runs the same materialize kernels with
 * their scratch in a fixed device array of SI_NOALLOC_SCRATCH_BYTES that the
 * library holds on every GPU where its module is loaded, until the process
 * exits.  Under CUDA's lazy module loading (the default) the array is
 * reserved by the first call on each device, which therefore needs that
 * much free memory itself (SI_ERR_OUT_OF_MEMORY if not): make that first
 * call, on a small problem, before the caller's own pool takes the memory.
 *   Same arguments, layouts, ownership and results as
 *   si_indexer_materialize (bf16 q, kc; fp32 w; device pointers).
 *   Returns SI_ERR_UNSUPPORTED, touching nothing, when the scratch need
 *   4*B*S*T*(H_I+1) + 256 bytes exceeds SI_NOALLOC_SCRATCH_BYTES, or T >
 *   16384.  Calls no cudaMalloc / cudaFree and nothing that allocates.
 *   Every call looks up the array's device address in the current context
 *   (cudaGetSymbolAddress, which allocates nothing once the module is
 *   loaded); make the first call on a device before any stream capture.
 *   All calls on a device share the array, which keeps the last call's
 *   contents (every word is overwritten before it is read); calls whose
 *   work overlaps on the same device race on it and must be serialised.
 */
#define SI_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
SI_API si_status si_indexer_materialize_noalloc(const void* q, const void* kc, const float* w,
                                                int B, int S, int T, int H_I, int D, int m, int k,
                                                int32_t* out_idx, float* out_score, void* stream);

/*
 * Two-stage indexer top-k: the V4.1-Flash indexer as its deployment notes
 * describe it ("two-level sparse attention", indexer section): a cheap
 * candidate stage picks, per query, n_keep blocks of `block` compressed keys
 * (the notes: 2048 blocks of 8), then the top-k of the candidates is kept
 * (the notes: 512).  Reading of what the pages leave open:
 *   - block j is keys j*block .. j*block+block-1 (floor(T/block) blocks);
 *     its pooled key is the mean of its keys rounded once to bf16;
 *   - a block competes for query t once all its keys are visible; the
 *     n_keep best by the indexer score of the pooled key are kept (all of
 *     them when fewer compete; ties to the lower block);
 *   - the candidates are the kept blocks' keys and the visible keys of the
 *     incomplete last block; the result is their top-k by the indexer score,
 *     exactly as si_indexer_topk orders and pads it.
 * With at most n_keep complete visible blocks the result is si_indexer_topk's.
 *   q [B,S,H_I,D] bf16, kc [B,T,D] bf16, w [B,S,H_I] fp32 (device);
 *   out_idx, out_score [B,S,k] (device, written; out_score required).
 * Supported: bf16 (opt->dtype 0 or opt NULL), D == 128, H_I == 64,
 * 1 <= k <= 2048, 1 <= n_keep <= 2048, 1 <= block <= 64; else
 * SI_ERR_UNSUPPORTED / SI_ERR_INVALID_ARGUMENT.  Rows are processed in
 * chunks of opt->query_chunk rows (0 = 16384); scratch of
 * si_two_stage_workspace_size() bytes comes from opt->workspace when given,
 * else it is allocated and freed on `stream`.  Asynchronous on `stream`.
 * Performance: a block size divisible by 8 (the notes' 8) loads each 8-key
 * run of candidates as one TMA box; one divisible by 4 as two smaller ones;
 * other sizes gather the candidate rows 16 bytes at a time, several times
 * slower.  kc must be 16-byte aligned (as for si_indexer_topk).
 */
SI_API si_status si_indexer_topk_two_stage(const void* q, const void* kc, const float* w, int B, int S, int T,
                                           int H_I, int D, int m, int k, int block, int n_keep,
                                           int32_t* out_idx, float* out_score, void* stream,
                                           const si_options* opt);

/* Scratch bytes of si_indexer_topk_two_stage (query_chunk 0 = 16384). */
SI_API size_t si_two_stage_workspace_size(int B, int S, int T, int block, int n_keep, int query_chunk);

/*
 * Sparse attention over the selected compressed latents: the consumer of the
 * top-k (StreamIndex abstract: the sparse attention kernel reads only the
 * entries the indexer selected).  Reading of the pages (the DeepSeek-V3.2
 * lineage the V4.1 page gives): each of the H heads of query t attends over
 * the k latents idx[b,t,:] of its sequence (index -1 is padding and is
 * skipped); a latent serves as the key (all Dk values) and as the value (its
 * first Dv values); the softmax runs over the selection only, with `scale`
 * (0 = 1/sqrt(Dk)).
 *   q   [B, S, H, Dk] bf16     kv  [B, T, Dk] bf16     idx [B, S, k] int32
 *   out [B, S, H, Dv] bf16 (written): sum_j softmax_j(scale q.kv_j) kv_j[:Dv]
 *   lse [B, S, H] fp32 (written): ln sum_j exp(scale q.kv_j)
 * A row with nothing selected gives out = 0 and lse = -inf.  Supported:
 * H == 64, Dk == 576, Dv == 512, k in {128, 256, 384, 512}; entries of idx
 * outside [-1, T) are treated as padding.  The softmax weights are rounded to
 * bf16 for the value product (their rounded sum normalises it).  Device
 * pointers, 16-byte aligned; asynchronous on `stream`; opt may be NULL (its
 * device_status is honoured, the other fields are ignored).
 */
SI_API si_status si_sparse_attention(const void* q, const void* kv, const int32_t* idx, int B, int S, int T,
                                     int H, int Dk, int Dv, int k, float scale, void* out, float* lse,
                                     void* stream, const si_options* opt);

/*
 * Decodes MXFP4 rows to bf16: codes [rows, D/2] bytes (value d in the low
 * nibble of byte d/2 when d is even, the high nibble when odd), E8M0 scales
 * [rows, D/32] (one per 32 values), out [rows, D] bf16; device pointers,
 * caller-owned; codes and out 16-byte aligned.  D a positive multiple of 32.
 * An E2M1 value times 2^(scale-127) is a bf16 value exactly for scales
 * <= 252; 253 and 254 can overflow to +-inf and 255 (NaN) gives NaN.
 * rows >= 0 (0: nothing).  Asynchronous on `stream`.  The streaming path's
 * key decode for SI_DTYPE_MXFP4_KEYS; also a conversion for callers.
 */
SI_API si_status si_mxfp4_to_bf16(const void* codes, const void* scales, int64_t rows, int D, void* out,
                                  void* stream);

/* Scratch bytes a call with these arguments needs (0 if none).  One function
 * serves two entry points, so it takes one argument more than the call it
 * sizes: materialize != 0 gives si_indexer_materialize's need,
 * 4*B*S*T*(H_I+1) + 256; materialize == 0 the streaming path's, which is
 * B*T*D*2 (+ alignment) for SI_DTYPE_MXFP4_KEYS and 0 for the others. */
SI_API size_t si_indexer_workspace_size(int B, int S, int T, int H_I, int D, int m, int k, int materialize,
                                 const si_options* opt);

/* Waits for `stream`, then returns SI_ERR_TIMEOUT (and clears the record) if
 * any kernel of this library that ran without its own si_options.device_status
 * word timed out in a bounded wait since the last call, else the stream's own
 * error state (SI_OK or SI_ERR_CUDA).  The record is per device and shared by
 * every stream and host thread on it; a caller that needs a per-call status
 * passes si_options.device_status instead. */
SI_API si_status si_device_status(void* stream);

SI_API const char* si_status_string(si_status s);
SI_API const char* si_last_error(void); /* thread-local; "" when none */
SI_API int si_version(void);            /* major*10000 + minor*100 + patch */

#ifdef __cplusplus
}
#endif
#endif /* STREAMING_TOP_H */
