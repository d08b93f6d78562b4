/*
 * fa.h -- C ABI of the B200 fused attention library (libfa.so).
 *
 * The operations follow fkl_python PR #6 ("fkl.flash_attention: FA-2 forward
 * with fused epilogue + compressed int8 KV cache"), Summary:
 *   - flash_attention(q, k, v, causal, epilogue=[ops])  -> fa_attention_fwd
 *   - compress_kv(k): per-token int8 + one fp32 scale   -> fa_compress_kv
 *   - the decode step s_q = 1 over the int8 cache        -> fa_attention_decode
 * and the C style of Foundry attention/README.md, API (fa_* calls over raw
 * buffers).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never frees them and keeps none of them after the call returns.
 *   - Every pointer must be 16-byte aligned and every row contiguous.
 *   - Work is enqueued asynchronously on the given stream (0 = legacy default
 *     stream).  Argument checks run on the host before any launch; a call that
 *     returns an error has enqueued nothing.
 *   - The library allocates only one small device status word per device, on
 *     first use, plus cached TMA descriptors.  It never prints and never
 *     throws across the ABI.
 *   - Bounded device waits: every spin on an mbarrier or flag in a kernel has
 *     a cycle budget; on expiry the kernel records FA_ERR_TIMEOUT in the
 *     status word and returns.  fa_check_device_error() reports it.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fa_stream_t; /* same type as cudaStream_t */

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID = 1,     /* bad argument: null pointer, shape, alignment, ... */
    FA_ERR_UNSUPPORTED = 2, /* well-formed, but no kernel for this combination */
    FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, descriptor) */
    FA_ERR_TIMEOUT = 4,     /* a bounded device wait gave up (see fa_check_device_error) */
    FA_ERR_WORKSPACE = 5    /* decode workspace missing or too small */
} fa_status;

typedef enum {
    FA_F32 = 0,  /* IEEE fp32 */
    FA_BF16 = 1, /* bfloat16 */
    FA_I8 = 2    /* int8 codes, with one fp32 scale per row (token, kv-head) */
} fa_dtype;

/* Epilogue ops (fkl_python PR #6, Summary: a list of elementwise ops that
 * the attention kernel itself applies to its output in registers; example
 * [Mul(2.0), Add(0.5)]).  They are applied to the normalised fp32
 * output in list order, each rounded to fp32 (no fused multiply-add), before
 * the cast to the output dtype.  Values are plain kernel arguments, so
 * changing them -- or the list's shape -- never compiles anything. */
typedef enum { FA_EPI_MUL = 1, FA_EPI_ADD = 2 } fa_epi_kind;
#define FA_MAX_EPILOGUE 8
typedef struct {
    int32_t op;  /* fa_epi_kind */
    float value;
} fa_epi_op;

/*
 * fa_compress_kv -- per-row int8 quantisation (fkl_python PR #6, Summary:
 * the KV cache compressed on the GPU to int8 codes per token, with one fp32
 * scale per token).
 *   x       [rows, d] FA_BF16 or FA_F32, row-major.  A row is one (token,
 *           kv-head) vector; K and V are compressed by separate calls.
 *   codes   [rows, d] int8 out;  scales [rows] fp32 out.
 * For each row: amax = max|x| (in fp32), s = amax / 127 (IEEE fp32 division),
 * c = clamp(round_half_even(x / s), -127, 127); an all-zero row gets s = 0
 * and zero codes.  Non-finite inputs give unspecified codes.
 * Requirements: rows >= 0 (0 enqueues nothing), 1 <= d <= 1024 with d % 16 == 0,
 * pointers 16-byte aligned.
 */
FA_API fa_status fa_compress_kv(const void *x, fa_dtype x_dtype, int64_t rows, int32_t d,
                         int8_t *codes, float *scales, fa_stream_t stream);

/*
 * Forward attention parameters (fkl_python PR #6, Summary: tensors laid out
 * as (batch*heads, seq, head_dim), accumulation in fp32, head sizes that are
 * multiples of 32).
 *
 * out = softmax(scale * q k^T + mask) v, then the epilogue chain.
 *
 * Dense layout (cu_seqlens_q == NULL):
 *     q, out [batch*hq, seqlen_q, d];  k, v [batch*hkv, seqlen_k, d].
 * Varlen layout (cu_seqlens_q != NULL; device int32 [batch+1], ascending,
 * cu[0] = 0; cu_seqlens_k NULL means the same as cu_seqlens_q):
 *     q, out [hq, total_q, d];  k, v [hkv, total_k, d]; sequence b owns rows
 *     cu[b] .. cu[b+1]-1 of every head plane.  total_q/total_k are the head
 *     plane heights and max_seqlen_q/k host-side upper bounds of the
 *     per-sequence lengths (used to size the grid; they must hold).
 * GQA: query head h reads KV head h / (hq / hkv); hq % hkv == 0.
 * Masks (per sequence with s_q queries and s_k keys; query i sits at key
 * position p = i + s_k - s_q, bottom-right aligned):
 *     causal != 0 keeps keys j <= p;  window > 0 keeps keys j > p - window;
 *     window <= 0 means no window.
 * A row with no visible key gets uniform weights over all s_k keys of its
 * sequence (the mean of V; zeros when s_k = 0) -- SKaiNET-transformers
 * PR #419, Summary: a sliding-window row whose band holds no key falls back
 * to the engine's uniform softmax.
 * dtypes: q_dtype FA_F32 (CUDA-core fp32 path; kv_dtype FA_F32 or FA_I8) or
 * FA_BF16 (tensor-core path; kv_dtype FA_BF16 or FA_I8).  FA_I8 K/V come
 * with k_scales/v_scales [batch*hkv, seqlen_k] dense or [hkv, total_k]
 * varlen, one fp32 scale per (token, kv-head) as fa_compress_kv writes them
 * (16-byte aligned on the BF16 path).  The kernels dequantise c * s on chip
 * (fkl_python PR #6, Summary): rounded to fp32 on the F32 path (relative
 * error at most 2^-24); on the BF16 path rounded to fp32 and then to bf16,
 * the tensor-core operand type.  out has q's dtype.
 * head_dim: F32 path any multiple of 32 up to 256; BF16 path 32, 64, 96, 128,
 * 160, 192, 224 or 256 (FA_BF16 or FA_I8 K/V).
 * A problem without keys (seqlen_k = 0, or varlen total_k = 0 with
 * cu_seqlens_k given) reads no K or V: k, v and the scales may be NULL.
 */
typedef struct {
    const void *q;
    const void *k;
    const void *v;
    void *out;
    const float *k_scales; /* FA_I8 only, else NULL */
    const float *v_scales; /* FA_I8 only, else NULL */
    int32_t q_dtype;       /* fa_dtype */
    int32_t kv_dtype;      /* fa_dtype */
    int32_t batch, hq, hkv, head_dim;
    int32_t seqlen_q, seqlen_k;          /* dense layout */
    const int32_t *cu_seqlens_q;         /* varlen layout (device) */
    const int32_t *cu_seqlens_k;
    int32_t total_q, total_k;            /* varlen head-plane heights */
    int32_t max_seqlen_q, max_seqlen_k;  /* varlen host-side bounds */
    int32_t causal;
    int32_t window;
    float softmax_scale;                 /* e.g. 1/sqrt(head_dim) */
    int32_t n_epilogue;                  /* 0 .. FA_MAX_EPILOGUE */
    fa_epi_op epilogue[FA_MAX_EPILOGUE];
} fa_fwd_params;

FA_API fa_status fa_attention_fwd(const fa_fwd_params *p, fa_stream_t stream);

/*
 * Single-query decode against a KV cache (fkl_python PR #6, Verification:
 * a one-query decode step over 256 int8-cached keys; Summary: the kernel
 * dequantises the compressed cache on chip, with no widened copy in global
 * memory).
 *   q        [batch*hq, d] bf16 (one query per sequence and head)
 *   k_cache, v_cache [batch*hkv, capacity, d], kv_dtype FA_I8 (with k_scales,
 *            v_scales [batch*hkv, capacity] fp32) or FA_BF16
 *   cache_seqlens  device int32 [batch]: sequence b attends to keys
 *            0 .. L_b-1 (the current token already appended), 0 <= L_b <= capacity;
 *            an L_b outside that range is clamped into it and reported by
 *            fa_check_device_error as FA_ERR_INVALID
 *   out      [batch*hq, d] bf16
 * The query sits at position L_b - 1, so every cached key is visible; a
 * window W > 0 keeps the last W.  L_b = 0 gives the epilogue applied to zeros.
 * Work is split along the keys: the 32-key tiles of all (sequence, KV head)
 * pairs are divided evenly among a persistent grid of warps, each of which
 * writes one partial (m, l, O) per pair it touches to the caller's workspace
 * (>= fa_decode_workspace_size bytes, 16-byte aligned, contents need no
 * initialisation); a merge kernel combines them.
 * max_seqlen: host-side upper bound of the L_b (0 means capacity; checked
 * against capacity only).  split_keys: 0, or a multiple of 256 -- the fewest
 * keys each warp is given (fewer, longer ranges).  capacity must be a
 * multiple of 32; cache entries at or past L_b may hold any bytes (they never
 * reach the result).
 * Supported: head_dim 32, 64, 96, 128 or 256 (FA_I8 and FA_BF16); any hq / hkv (a group
 * of more than 8 query heads is served in passes of at most 8 heads, each
 * reading the KV head's cache once).
 */
typedef struct {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const float *k_scales;
    const float *v_scales;
    const int32_t *cache_seqlens;
    void *out;
    int32_t kv_dtype; /* fa_dtype: FA_I8 or FA_BF16 */
    int32_t batch, hq, hkv, head_dim, capacity;
    int32_t max_seqlen;
    int32_t window;
    float softmax_scale;
    int32_t split_keys; /* keys per split, multiple of 256; 0 = library choice */
    int32_t n_epilogue;
    fa_epi_op epilogue[FA_MAX_EPILOGUE];
    void *workspace;
    size_t workspace_bytes;
} fa_decode_params;

/* Bytes of decode workspace at these sizes (any hkv dividing hq; the count
 * of SMs of the current device enters it). */
FA_API size_t fa_decode_workspace_size(int32_t batch, int32_t hq, int32_t capacity, int32_t head_dim);

FA_API fa_status fa_attention_decode(const fa_decode_params *p, fa_stream_t stream);

/*
 * fa_attention_decode_paged -- fa_attention_decode over a paged cache, so a
 * serving loop hands the kernel its cache pages in place instead of copying
 * each sequence's prefix into a contiguous buffer (SKaiNET-transformers
 * PR #419, Summary: the positional KV caches give the kernel views of the
 * cached prefix where it lies, with no per-token copy).
 *   k_cache, v_cache  page pools [num_pages, hkv, page_size, d] (FA_I8 codes
 *                     with k_scales, v_scales [num_pages, hkv, page_size], or FA_BF16)
 *   block_table       device int32 [batch, max_pages]: key j of sequence b
 *                     is token j % page_size of page block_table[b][j / page_size]
 * Everything else as fa_attention_decode, with p->capacity the logical
 * capacity max_pages * page_size (cache_seqlens <= capacity) and the same
 * workspace size.  Only the pages holding attended keys are read; other
 * table entries may hold anything.  page_size is a multiple of 32 and
 * num_pages * hkv * page_size < 2^31.  A page id outside [0, num_pages) is
 * reported by fa_check_device_error as FA_ERR_INVALID; the kernel reads page
 * 0 in its place (never outside the pool) and that sequence's output is
 * meaningless.  Results equal fa_attention_decode's on the same keys bit for
 * bit (same split, same arithmetic).
 */
typedef struct {
    const int32_t *block_table;
    int32_t max_pages;   /* row length of block_table */
    int32_t page_size;   /* tokens per page, multiple of 32 */
    int32_t num_pages;   /* pages in each pool */
} fa_kv_pages;

FA_API fa_status fa_attention_decode_paged(const fa_decode_params *p, const fa_kv_pages *pages,
                                           fa_stream_t stream);

/*
 * fa_attention_fwd_paged -- fa_attention_fwd with K/V read from page pools
 * through a block table (SKaiNET-transformers PR #419, Summary: copy-free
 * K/V views for prefill as well as decode): e.g. a chunk of new queries per
 * sequence attending to that sequence's whole cached prefix, without copying
 * the prefix out of its pages.
 *   q, out   dense [batch*hq, seqlen_q, d] (cu_seqlens_q NULL) or varlen
 *            [hq, total_q, d] with cu_seqlens_q / max_seqlen_q, as for
 *            fa_attention_fwd; bf16
 *   k, v     page pools [num_pages, hkv, page_size, d] (FA_BF16, or FA_I8
 *            codes with k_scales, v_scales [num_pages, hkv, page_size])
 *   cu_seqlens_k  device int32 [batch+1]: sequence b has
 *            cu_seqlens_k[b+1] - cu_seqlens_k[b] keys, key j in token
 *            j % page_size of page block_table[b][j / page_size]
 * Masks, GQA, the empty-band rule and the epilogue as fa_attention_fwd
 * (query i of a sequence with s_q queries and s_k keys sits at key position
 * i + s_k - s_q).  page_size is a multiple of 128 (a 128-key tile never
 * crosses a page); seqlen_k, total_k and max_seqlen_k are not used.  A page id
 * outside [0, num_pages) reads page 0 and is reported by
 * fa_check_device_error as FA_ERR_INVALID.  Results equal fa_attention_fwd's
 * on the same keys in a contiguous layout bit for bit.
 */
FA_API fa_status fa_attention_fwd_paged(const fa_fwd_params *p, const fa_kv_pages *pages, fa_stream_t stream);

/*
 * fa_attention_fwd_lse -- fa_attention_fwd (bf16 tensor-core path) that also
 * returns, per output row, the natural log-sum-exp of the row's scaled
 * scores over its visible keys: a partial result that fa_attention_merge can
 * combine with others over disjoint key sets (the per-step (m, l, O) state
 * of a split or ring computation -- kernbench2 commit message, ADR-0060 (long context)).
 *   lse  [batch*hq*seqlen_q] fp32 (dense) or [hq*total_q] (varlen), the row
 *        numbering of out
 * A row without visible keys gets out = the epilogue applied to 0 and
 * lse = -inf (no uniform fallback: such a row weighs nothing in a merge).
 * Partial results meant for merging should carry no epilogue.
 */
FA_API fa_status fa_attention_fwd_lse(const fa_fwd_params *p, float *lse, fa_stream_t stream);

/*
 * fa_attention_fwd_acc -- fa_attention_fwd_lse and fa_attention_merge in one
 * pass: the attention of q over this call's keys is merged, row by row, into
 * an fp32 accumulator inside the kernel's epilogue, so a result built up over
 * several key blocks (the steps of a ring / context-parallel prefill --
 * kernbench2 commit message, ADR-0060 (long context): an online-softmax
 * merge at every ring step) costs no separate merge pass.
 *   o_acc   [rows of out, head_dim] fp32 (out's row numbering), 16-byte aligned
 *   lse_acc [rows of out] fp32: natural log-sum-exp of the scaled scores seen
 *           so far (-inf: none), 16-byte aligned
 *   flags   FA_ACC_FIRST: the accumulator holds nothing yet and is not read
 *           (it is written as if it had been o = 0, lse = -inf);
 *           FA_ACC_LAST: the merged rows are written to p->out, after the
 *           epilogue, instead of back to the accumulator (left unchanged)
 * p->out is used only with FA_ACC_LAST (may be NULL otherwise), and the
 * epilogue applies only there.  A row without visible keys merges nothing.
 * BF16 path (q FA_BF16, K/V FA_BF16 or FA_I8) only: other q types give
 * FA_ERR_UNSUPPORTED.
 */
#define FA_ACC_FIRST 1
#define FA_ACC_LAST 2
FA_API fa_status fa_attention_fwd_acc(const fa_fwd_params *p, float *o_acc, float *lse_acc, int32_t flags,
                                      fa_stream_t stream);

/*
 * fa_attention_merge -- fold a partial attention result into an accumulator:
 *   lse = log(e^lse_acc + e^lse_part)
 *   o_acc = o_acc e^(lse_acc - lse) + o_part e^(lse_part - lse)
 * per row (lse_acc = -inf and o_acc = 0 start an empty accumulator; two
 * empty rows stay empty).  o_part NULL merges nothing (only writes out).
 *   o_acc     [rows, head_dim] fp32, updated in place;  lse_acc [rows] fp32
 *   o_part    [rows, head_dim] part_dtype (FA_BF16 or FA_F32);  lse_part [rows]
 *   out       optional [rows, head_dim] out_dtype (FA_BF16 or FA_F32): the
 *             merged rows after the epilogue (the last merge of a sequence)
 * head_dim a multiple of 32 up to 256; pointers 16-byte aligned.
 */
typedef struct {
    float *o_acc;
    float *lse_acc;
    const void *o_part;
    int32_t part_dtype;
    const float *lse_part;
    int64_t rows;
    int32_t head_dim;
    void *out;
    int32_t out_dtype;
    int32_t n_epilogue;
    fa_epi_op epilogue[FA_MAX_EPILOGUE];
} fa_merge_params;

FA_API fa_status fa_attention_merge(const fa_merge_params *p, fa_stream_t stream);

/*
 * fa_kv_append -- write one new token per sequence into a decode KV cache,
 * quantising on the way in (FlashRT QKV Cache RoPE, Kernels: the
 * decode_k_norm_rope_kvwrite_devpos_bf16 kernel reads its cache slot from a
 * device-side int32 position, so a captured decode graph can replay it; here
 * without the norm and rotation, and with the int8 cache of fkl_python PR #6,
 * Summary: per-token int8 codes with one fp32 scale per token).
 *   k_new, v_new  [batch*hkv, d] x_dtype (FA_BF16 or FA_F32): the new token's
 *                 K and V rows, row u = b * hkv + g
 *   k_cache, v_cache [batch*hkv, capacity, d] cache_dtype: FA_I8 codes (with
 *                 k_scales, v_scales [batch*hkv, capacity] fp32) or FA_BF16
 *   cur_pos       device int32 [batch]: the slot written for sequence b
 *   cache_seqlens optional device int32 [batch] (NULL: untouched): set to
 *                 cur_pos[b] + 1, the length a following fa_attention_decode
 *                 attends to; it must not overlap cur_pos
 * Row u of K goes to cache row u * capacity + cur_pos[b] as int8 codes and
 * scale computed exactly as fa_compress_kv computes them (bit-identical), or
 * as bf16 (exact for bf16 input, round to nearest even for fp32).  Nothing
 * else in the caches changes.  Because the slot is read on the device, one
 * captured CUDA graph can append and decode step after step while a kernel
 * (or copy) in the same graph advances cur_pos.  A cur_pos[b] outside
 * [0, capacity) skips sequence b's rows (and its cache_seqlens entry) and is
 * reported by fa_check_device_error as FA_ERR_INVALID.  As with every entry
 * point, the first call on a device allocates the status word: make it
 * before any stream capture.
 * Requirements: 16 <= d <= 1024, d % 16 == 0; pointers 16-byte aligned;
 * capacity >= 1.  batch * hkv = 0 enqueues nothing.
 */
typedef struct {
    const void *k_new;
    const void *v_new;
    int32_t x_dtype;      /* fa_dtype: FA_BF16 or FA_F32 */
    void *k_cache;
    void *v_cache;
    float *k_scales;      /* FA_I8 cache only, else NULL */
    float *v_scales;
    int32_t cache_dtype;  /* fa_dtype: FA_I8 or FA_BF16 */
    const int32_t *cur_pos;
    int32_t *cache_seqlens;
    int32_t batch, hkv, head_dim, capacity;
} fa_kv_append_params;

FA_API fa_status fa_kv_append(const fa_kv_append_params *p, fa_stream_t stream);

/*
 * fa_kv_append_paged -- fa_kv_append into page pools [num_pages, hkv,
 * page_size, d] (scales [num_pages, hkv, page_size]) through the block table
 * of fa_attention_decode_paged: the slot cur_pos[b] is token cur_pos[b] %
 * page_size of page block_table[b][cur_pos[b] / page_size]; p->capacity is
 * max_pages * page_size.  A page id outside [0, num_pages) skips that
 * sequence's rows and is reported like an out-of-range slot.
 */
FA_API fa_status fa_kv_append_paged(const fa_kv_append_params *p, const fa_kv_pages *pages,
                                    fa_stream_t stream);

/*
 * fa_attention_decode_noalloc -- fa_attention_decode for callers that cannot
 * allocate device memory when they call.  The paper has no counterpart: this
 * entry point exists for callers such as a plug-in inside a serving runtime
 * that owns every device byte through its own pre-planned arena (allocating
 * outside it is forbidden or breaks its accounting), or code that must not
 * trigger the implicit device synchronisation a cudaMalloc can cause.
 *
 * Same parameters and results as fa_attention_decode, except that
 * p->workspace and p->workspace_bytes are ignored: the per-split partials go
 * to a scratch array of FA_DECODE_NOALLOC_SCRATCH_BYTES (8 MiB) built into
 * the library, which every device that loads the library holds until the
 * process exits.  The call allocates nothing (no cudaMalloc, no library
 * allocator).
 *   - Limit: the scratch holds the per-sequence tile plan ((batch + 1) * 4
 *     bytes), one partial record per (sequence, KV head) and one per worker
 *     warp, each hq / hkv * (head_dim + 2) * 4 bytes.  The library uses as
 *     many workers as fit (up to its usual count); a problem where
 *     batch * hq * (head_dim + 2) * 4 bytes leave no room for one CTA of 4
 *     workers returns FA_ERR_WORKSPACE and enqueues nothing.  Only the int8
 *     cache (FA_I8) is supported.
 *   - The first call on each device looks up the scratch array's device
 *     address (with that device current); make that first call before any
 *     stream capture.
 *   - All calls on a device share the scratch and it keeps the last call's
 *     contents (nothing in it needs clearing).  Calls that overlap on the GPU
 *     race on it: serialise them (one stream, or events between streams).
 *   - A bounded device wait that gives up inside this call, or a cache
 *     length outside [0, capacity], is recorded in a status word of this
 *     entry point's own (a statically allocated device word: the library's
 *     shared one is allocated on first use).  fa_check_device_error reads and
 *     clears both words, allocating nothing, and reports FA_ERR_TIMEOUT or
 *     FA_ERR_INVALID as for the other entry points.
 */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
FA_API fa_status fa_attention_decode_noalloc(const fa_decode_params *p, fa_stream_t stream);

/* Static text for a status code (never NULL). */
FA_API const char *fa_status_string(fa_status s);

/*
 * TurboQuant KV cache compression (the C attention library's README,
 * "TurboQuant KV Cache Compression"): a K or V row x of head size d is
 * rotated, y = H (s * x) / sqrt(d) with H the Sylvester-ordered Hadamard
 * matrix and s random +-1 signs applied before it, normalised by its L2
 * norm, u = y / ||x||, and each u_i replaced by the b-bit index of the
 * nearest level of the Lloyd-Max quantiser of the Beta(d/2, d/2) law of
 * (u + 1) / 2 (a tie goes to the lower level); the codes are bit-packed,
 * channel i at bits [i b, i b + b) of the row's little-endian bit stream,
 * beside one fp32 norm per row.  A row reads back as
 * x_hat = s * (H (||x|| level[code])) / sqrt(d).  K4/V2 at d = 64 is 56
 * bytes per token and KV head against 512 in fp32 (the page's 9.14x).
 *
 * fa_tq_codebook -- host function: the 2^bits levels in u-space, ascending
 * and antisymmetric, into levels[] (host memory).  4 <= head_dim <= 2^20,
 * head_dim even; 1 <= bits <= 8.  Computed in double by Lloyd's iteration
 * on a 2^20-interval quadrature of the density (1 - u^2)^(d/2 - 1).
 */
FA_API fa_status fa_tq_codebook(int32_t head_dim, int32_t bits, float *levels);

/*
 * fa_tq_compress -- rows of K or V into packed codes and norms.
 *   x       [rows, head_dim] x_dtype (FA_BF16 or FA_F32)
 *   signs   device [head_dim] fp32, each +1 or -1 (the rotation)
 *   levels  device [2^bits] fp32 (fa_tq_codebook(head_dim, bits))
 *   codes   [rows, head_dim * bits / 8] uint8;  norms [rows] fp32
 * head_dim 64 or 128; bits 2, 3 or 4; every pointer 16-byte aligned; the
 * decisions are taken in fp32 (a value within rounding of a cell edge may
 * land on either side).  rows = 0 enqueues nothing.
 */
typedef struct {
    const void *x;
    int32_t x_dtype;
    int64_t rows;
    int32_t head_dim;
    int32_t bits;
    const float *signs;
    const float *levels;
    uint8_t *codes;
    float *norms;
} fa_tq_compress_params;

FA_API fa_status fa_tq_compress(const fa_tq_compress_params *p, fa_stream_t stream);

/*
 * fa_tq_attention_decode -- s_q = 1 attention of every query head over a
 * TurboQuant cache, without rebuilding K or V: scores are
 * ||k|| (R q) . level[code] with R the rotation, the V side is accumulated
 * in the rotated basis and rotated back once per output row.
 *   q          [batch*hq, head_dim] bf16;  out [batch*hq, head_dim] bf16
 *   k_codes    [batch*hkv, capacity, head_dim*k_bits/8] uint8, k_norms
 *              [batch*hkv, capacity] fp32 (fa_tq_compress of the K rows);
 *              v_codes / v_norms likewise with v_bits
 *   k_levels, v_levels  device [2^bits] fp32, ascending and antisymmetric
 *              (level[n-1-i] = -level[i], as fa_tq_codebook returns them: the
 *              K side is looked up from the upper half, mirrored for the
 *              lower);  signs device [head_dim] fp32 (one rotation for K and V)
 *   cache_seqlens device int32 [batch]: keys 0 .. L_b - 1 are attended; a
 *              value outside [0, capacity] is clamped and reported by
 *              fa_check_device_error as FA_ERR_INVALID; L_b = 0 gives the
 *              epilogue of 0
 *   workspace  device, >= fa_tq_decode_workspace_size() bytes (partials of
 *              the key splits), 16-byte aligned
 * head_dim 64 or 128; k_bits, v_bits 2..4; hq / hkv in {1, 2, 4, 8}.
 */
typedef struct {
    const void *q;
    const uint8_t *k_codes;
    const float *k_norms;
    const uint8_t *v_codes;
    const float *v_norms;
    const float *k_levels;
    const float *v_levels;
    const float *signs;
    const int32_t *cache_seqlens;
    int32_t batch;
    int32_t hq;
    int32_t hkv;
    int32_t head_dim;
    int32_t capacity;
    int32_t k_bits;
    int32_t v_bits;
    float softmax_scale;
    void *out;
    void *workspace;
    size_t workspace_bytes;
    int32_t n_epilogue;
    fa_epi_op epilogue[FA_MAX_EPILOGUE];
} fa_tq_decode_params;

FA_API size_t fa_tq_decode_workspace_size(int32_t batch, int32_t hq, int32_t head_dim, int32_t capacity);
FA_API fa_status fa_tq_attention_decode(const fa_tq_decode_params *p, fa_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * words (the shared one and fa_attention_decode_noalloc's own):
 * FA_ERR_TIMEOUT if a bounded wait in any kernel gave up since the last
 * check, FA_ERR_INVALID if a kernel met a device-side argument out of range
 * (fa_kv_append's cur_pos, a paged call's page id, a decode cache length),
 * FA_ERR_CUDA if the synchronisation itself failed, else FA_OK.  It
 * allocates nothing: before the first launch on a device there is nothing
 * to read.
 */
FA_API fa_status fa_check_device_error(fa_stream_t stream);

/*
 * Diagnostic: launches one tiny kernel that waits on an mbarrier no thread
 * ever arrives on, with a budget of `budget_cycles` SM cycles (clamped to
 * [1e3, 1e9]).  The wait runs out, the kernel records FA_ERR_TIMEOUT and
 * returns; fa_check_device_error() must then report FA_ERR_TIMEOUT.  Used to
 * test the watchdog path without faulting or hanging the device.
 */
FA_API fa_status fa_selftest_watchdog(uint64_t budget_cycles, fa_stream_t stream);

/* Number of distinct kernel instantiations launched so far by this process
 * (the epilogue never adds one: values and list length are runtime data). */
FA_API int32_t fa_kernel_variants_used(void);

/* Total kernel launches made by this library in this process (all devices);
 * a diagnostic for counting launches inside a timed region. */
FA_API int64_t fa_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
