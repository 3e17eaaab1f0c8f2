/*
 * libmqa — single-token incremental-decode attention over a KV cache, for
 * NVIDIA B200 (sm_100a).  Multi-Query Attention (h query heads share one K/V
 * head), Grouped-Query Attention (g K/V heads, each shared by h/g query heads)
 * and Multi-Head Attention (g = h) are one computation with one parameter g.
 *
 * The computation, from the incremental decode step of "Fast Transformer
 * Decoding: One Write-Head is All You Need" (the velog paper review, §3
 * "Multi Query Attention", MultiquerySelfAttentionIncremental; §2.4 for the
 * per-head MHA form) with the projections left to the caller:
 *
 *   new_K = concat(prev_K, k_new)                       -> mqa_kv_append
 *   logits = einsum("bhk,bmk->bhm", q, new_K) * scale   -> mqa_decode
 *   weights = softmax(logits) over each sequence's valid rows
 *   o = einsum("bhm,bmv->bhv", weights, new_V)
 *
 * Grouping follows the GQA blog ("GQA、MQA、MLA", section "第三站: GQA"):
 * query head i reads K/V head j = i / (h/g).  The scale is the 1/sqrt(d_h) of
 * the study notes' §1 formula when the caller wants it; pass 1.0 when q is
 * already scaled (the paper's code has no scale).
 *
 * Conventions shared by every call
 *  - All pointers named "device" are CUDA device pointers on the current
 *    device, owned by the caller, 16-byte aligned, and not aliased with each
 *    other.  The library allocates nothing and keeps no state between calls
 *    besides per-device attribute caches.
 *  - Tensors are dense and row-major in the stated shapes.  q, the caches and
 *    o share one element type (mqa_dtype_t); arithmetic is fp32 throughout.
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream).
 *    Arguments are checked before anything is launched: a failed check
 *    returns MQA_ERR_INVALID_ARG or MQA_ERR_UNSUPPORTED and launches nothing.
 *    A launch failure returns MQA_ERR_CUDA.  Nothing traps, nothing throws.
 *  - Values read on the device (lens, pos) are clamped or skipped, never
 *    trusted: the offending case sets a bit in *status_flags (a caller-owned
 *    device int32, may be NULL) with an atomic OR.  The library never clears
 *    it; the caller zeroes it when it wants a fresh reading.
 */
#ifndef LIBMQA_MQA_H
#define LIBMQA_MQA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MQA_API __attribute__((visibility("default")))
#else
#define MQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MQA_OK = 0,
  MQA_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or combination */
  MQA_ERR_UNSUPPORTED = 2,   /* valid, but not built (e.g. head size 96)      */
  MQA_ERR_CUDA = 3           /* a CUDA call or launch failed                  */
} mqa_status_t;

typedef enum {
  MQA_F32 = 0,               /* float32 storage                                */
  MQA_BF16 = 1               /* bfloat16 storage, round-to-nearest-even output */
} mqa_dtype_t;

/* Bits of *status_flags. */
#define MQA_FLAG_LEN_CLAMPED 1 /* a lens[b] was outside [1, m_max]; clamped     */
#define MQA_FLAG_POS_SKIPPED 2 /* a pos[b] was outside [0, m_max); not written  */
#define MQA_FLAG_PIPE_TIMEOUT 4 /* a tensor-core pipeline wait ran out; the
                                   outputs of that call are not valid           */

/* Kernel path of mqa_decode_ex. */
typedef enum {
  MQA_PATH_AUTO = 0,         /* tensor cores when bf16, d_k and d_v each 64
                                or 128, h/g <= 64; else CUDA cores           */
  MQA_PATH_SIMT = 1,         /* CUDA-core FFMA path (any dtype, h/g*d <= 4096) */
  MQA_PATH_TCGEN05 = 2       /* tcgen05 tensor-core path (bf16, d_k and d_v
                                each 64 or 128, h/g <= 64)                    */
} mqa_path_t;

typedef struct {
  int path;                  /* mqa_path_t                                     */
  int num_ctas;              /* persistent CTAs; 0 = SM count x resident CTAs  */
  int window;                /* local attention: attend only to the newest
                                `window` valid rows of each sequence, rows
                                [max(0, lens[b] - window), lens[b]); 0 = all
                                rows.  "Fast Transformer Decoding" study notes
                                §6.1 (the decoder's window: the current
                                position and the 31 before it, window = 32)
                                and §6.4 (local attention combined with MQA).
                                Must be >= 0.                                  */
} mqa_decode_opts_t;

/* Largest number of persistent CTAs a decode may use; sizes the workspace. */
#define MQA_MAX_CTAS 2048

/*
 * mqa_kv_append — write one step's K and V into the cache ("one write-head").
 *
 * Source: the velog paper review, §3 MultiquerySelfAttentionIncremental,
 * new_K = concat([prev_K, expand_dims(k_new)]) and the same for V; with a
 * fixed-size cache the concat is a write at row pos[b].
 *
 *   k_cache  device [b, m_max, g, d_k]   written at rows pos[b] only
 *   v_cache  device [b, m_max, g, d_v]   written at rows pos[b] only
 *   k_new    device [b, g, d_k]          read
 *   v_new    device [b, g, d_v]          read
 *   pos      device int32 [b]            row to write for each sequence
 *   status_flags  device int32 or NULL   MQA_FLAG_POS_SKIPPED when some pos[b]
 *                                        is outside [0, m_max); that sequence
 *                                        is left untouched
 * The copy is bitwise.  b = 0 is a no-op returning MQA_OK.  Errors:
 * MQA_ERR_INVALID_ARG for NULL pointers, negative sizes, a row size
 * (d * element size) that is not a multiple of 16 bytes, or misalignment.
 * Intended order within a step: append at pos = old length, then decode with
 * lens = old length + 1 (the review's step concatenates before attending).
 */
MQA_API mqa_status_t mqa_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                           const int32_t* pos, int b, int m_max, int g, int d_k, int d_v,
                           mqa_dtype_t dtype, int32_t* status_flags, cudaStream_t stream);

/*
 * mqa_decode_workspace_size — bytes of device scratch mqa_decode needs.
 * Pure host arithmetic (no CUDA call).  The workspace holds, per split of a
 * sequence's rows, the normalised partial output (fp32 [h/g, d_v]) and its
 * log-sum-exp, plus two ints per (sequence, K/V head).  Returns 0 for
 * invalid sizes.
 */
MQA_API size_t mqa_decode_workspace_size(int b, int h, int g, int d_v);

/*
 * mqa_decode — attention of each sequence's newest query over its cache.
 *
 * Source: the velog paper review, §3 (MQA) and §2.4 (MHA) incremental code,
 * logits = einsum("bhk,bmk->bhm"), softmax, o = einsum("bhm,bmv->bhv"); the
 * scaled softmax of the study notes §1; GQA grouping of the GQA blog.
 *
 *   o        device [b, h, d_v]          written (every element)
 *   q        device [b, h, d_k]          read
 *   k_cache  device [b, m_max, g, d_k]   rows t < lens[b] read; others never
 *   v_cache  device [b, m_max, g, d_v]   rows t < lens[b] read; others never
 *   lens     device int32 [b]            valid rows per sequence; values
 *                                        outside [1, m_max] are clamped
 *                                        (<= 0 gives an all-zero output row)
 *                                        and set MQA_FLAG_LEN_CLAMPED
 *   scale    multiplies q . k (finite)
 *   workspace        device scratch of at least
 *                    mqa_decode_workspace_size(b, h, g, d_v) bytes, 256-byte
 *                    aligned; contents on entry do not matter; calls that
 *                    share a workspace must be ordered on one stream
 *   status_flags     device int32 or NULL (see above)
 * Supported: h % g == 0, d_k and d_v in {32, 64, 128}, in any pairing (the
 * paper's per-head key size k and value size v are independent).  The SIMT
 * path takes h/g * d_k <= 4096 and h/g * d_v <= 4096; the tensor-core path
 * bf16 with d_k and d_v each 64 or 128 (any pairing) and h/g <= 64, which the
 * automatic choice then takes.  b = 0 is a no-op returning MQA_OK.
 * Errors: MQA_ERR_INVALID_ARG (NULL pointer, h % g != 0, non-finite scale,
 * workspace too small or misaligned), MQA_ERR_UNSUPPORTED (head sizes or
 * group widths not built), MQA_ERR_CUDA (launch failure).
 */
MQA_API mqa_status_t mqa_decode(void* o, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* lens, int b, int h, int g, int m_max, int d_k, int d_v,
                        float scale, mqa_dtype_t dtype, void* workspace, size_t workspace_bytes,
                        int32_t* status_flags, cudaStream_t stream);

/* mqa_decode with an explicit kernel path and CTA count (opts may be NULL,
 * which is mqa_decode).  Requesting a path that cannot serve the arguments
 * returns MQA_ERR_UNSUPPORTED. */
MQA_API mqa_status_t mqa_decode_ex(void* o, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* lens, int b, int h, int g, int m_max, int d_k, int d_v,
                           float scale, mqa_dtype_t dtype, void* workspace, size_t workspace_bytes,
                           int32_t* status_flags, const mqa_decode_opts_t* opts, cudaStream_t stream);

/*
 * mqa_decode_append — one whole incremental step: append, then attend.
 *
 * Source: the velog paper review, §3 MultiquerySelfAttentionIncremental:
 * new_K = concat(prev_K, k_new), new_V likewise, then the attention of
 * mqa_decode over new_K/new_V.  Here lens[b] counts the rows after the
 * append, so the step's K/V row goes to row lens[b]-1.  Same result as
 * mqa_kv_append(pos = lens-1) followed by mqa_decode(lens), in one launch:
 * the CTA that loads a sequence's last tile first writes the new row into the
 * cache, then attends over it.
 *
 *   k_cache, v_cache  device [b, m_max, g, d_k], [b, m_max, g, d_v]
 *                     read, and row lens[b]-1 written
 *   k_new, v_new      device [b, g, d_k], [b, g, d_v]   read
 *   other arguments as for mqa_decode_ex; lens outside [1, m_max] are clamped
 *   and flagged as there (the row then goes to the clamped length minus one;
 *   a sequence whose clamped length is 0 writes nothing and outputs zeros).
 * Errors as for mqa_decode_ex, plus MQA_ERR_INVALID_ARG for NULL or
 * misaligned k_new / v_new.
 */
MQA_API mqa_status_t mqa_decode_append(void* o, const void* q, void* k_cache, void* v_cache, const void* k_new,
                                       const void* v_new, const int32_t* lens, int b, int h, int g, int m_max,
                                       int d_k, int d_v, float scale, mqa_dtype_t dtype, void* workspace,
                                       size_t workspace_bytes, int32_t* status_flags,
                                       const mqa_decode_opts_t* opts, cudaStream_t stream);

/* Size of the device array that mqa_decode_noalloc uses as its scratch. */
#define MQA_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * mqa_decode_noalloc — mqa_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a deployment variant of
 * the same computation, not a step of the method.
 *
 * Who needs it: code that must not call cudaMalloc or any other allocator —
 * a plugin whose host application owns all device memory, a runtime with a
 * memory pool fixed at start-up, or a call site where an allocation could
 * synchronise the device or fail at a point where failure is not allowed.
 * Instead of a caller-provided workspace, the split partials live in a
 * device array of MQA_NOALLOC_SCRATCH_BYTES (16 MiB) that the library
 * defines; every GPU on which the library is loaded holds that array until
 * the process exits.  The call allocates nothing.
 *
 * Arguments, results, flags and errors are those of mqa_decode without the
 * workspace pair; the caller still provides o, q, the caches and lens.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current).  Make that first call before any
 *    stream capture on the device.  Under lazy module loading (the default
 *    since CUDA 12) that first call may also be what loads the library's
 *    device code on the device, which reserves the 16 MiB array there; if
 *    the device has no room left, the call returns MQA_ERR_CUDA.  A caller
 *    that wants no surprise later makes one warm-up call at start-up.
 *  - The array holds the partials of the last call; every value a call reads
 *    back from it was written earlier in the same call, so nothing in it has
 *    to start at zero.
 *  - All calls on a device share the one array: calls whose work can overlap
 *    on the GPU (different streams without ordering, several host threads)
 *    race on it and give wrong results.  Order them on one stream.
 *  - Shapes whose partials cannot fit even with a single CTA (roughly
 *    b * g * h/g * (d_v + 1) * 4 bytes above 16 MiB) are rejected with
 *    MQA_ERR_INVALID_ARG before anything is launched; otherwise the number of
 *    CTAs is lowered until the partials fit.
 */
MQA_API mqa_status_t mqa_decode_noalloc(void* o, const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* lens, int b, int h, int g, int m_max, int d_k, int d_v,
                                        float scale, mqa_dtype_t dtype, int32_t* status_flags,
                                        cudaStream_t stream);

/*
 * mqa_decode_beam — one decode step of W beams per sequence that share the
 * sequence's prefix (beam search).
 *
 * Source: the study notes on "Fast Transformer Decoding", §6.2 and §6.4, time
 * a beam-4 decoder (MQA 32 us vs MHA 203 us per token; local MQA 16 us); the
 * pages give no formula.  Reading: beam w of sequence s attends over the
 * prefix rows 0..prefix_lens[s]-1 of sequence s followed by its own suffix
 * rows 0..suffix_lens[s*W+w]-1 (the tokens that beam generated).  One pass:
 * the prefix is read once for all W beams, its K/V tiles feeding the W beams'
 * query heads of a group together (W*h/g query rows per tile), and then each
 * beam's suffix rows, which count for that beam's heads only; sequences split
 * between CTAs are merged with log-sum-exp weights afterwards.
 *
 *   o            device [b, W, h, d_v]   written
 *   q            device [b, W, h, d_k]
 *   prefix_k/v   device [b, m_p, g, d]   prefix_lens device int32 [b]
 *   suffix_k/v   device [b*W, m_s, g, d] suffix_lens device int32 [b*W]
 *   workspace    device, mqa_decode_beam_workspace_size(b, W, h, g, d_v)
 *                bytes, 256-byte aligned; contents on entry do not matter
 *
 * Lengths are clamped to [0, m_p] and [0, m_s] (MQA_FLAG_LEN_CLAMPED); a beam
 * with no rows gets a zero row.  Only bf16 with d_k = d_v = 128 and
 * W*h/g <= 64 is built (MQA_ERR_UNSUPPORTED otherwise).  Append the step's
 * K/V to the suffix caches first (mqa_kv_append with the suffix caches).
 */
MQA_API size_t mqa_decode_beam_workspace_size(int b, int W, int h, int g, int d_v);
MQA_API mqa_status_t mqa_decode_beam(void* o, const void* q, const void* prefix_k, const void* prefix_v,
                                     const int32_t* prefix_lens, const void* suffix_k, const void* suffix_v,
                                     const int32_t* suffix_lens, int b, int W, int h, int g, int m_p, int m_s,
                                     int d_k, int d_v, float scale, mqa_dtype_t dtype, void* workspace,
                                     size_t workspace_bytes, int32_t* status_flags, cudaStream_t stream);

/*
 * mqa_prefill — batched (prefill) attention: every position of every
 * sequence attends to the keys of its own sequence.
 *
 * Source: the paper review of "Fast Transformer Decoding", §2.3 Multi-head
 * Attention (Batched): logits = einsum("bhnk,bhmk->bhnm", Q, K),
 * weights = softmax(logits + mask), O = einsum("bhnm,bhmv->bhnv", weights, V),
 * with the K/V head axis removed as in §3 (h/g query heads per K/V head); the
 * study notes on the same paper, §1 and §10, describe prefill as the whole
 * prompt at once under a causal mask.  Here the mask is causal (causal = 1:
 * position t sees keys 0..t of its sequence) or absent (causal = 0: all keys
 * of the sequence), and sequences are packed without padding:
 *
 *   o           device [total, h, d_v]   written for every row of a sequence
 *   q           device [total, h, d_k]
 *   k, v        device [total, g, d_k], [total, g, d_v]
 *   cu_seqlens  device int32 [b+1]: sequence s holds rows
 *               cu_seqlens[s] .. cu_seqlens[s+1]-1 (non-decreasing, from 0)
 *   max_seqlen  host: the longest sequence; the launch covers that many
 *               positions per sequence
 *   scale       multiplies the logits (e.g. 1/sqrt(d_k))
 *
 * Row-major, contiguous, 16-byte aligned, caller-owned.  Only bf16 with
 * d_k = d_v = 128 and h/g dividing 128 is built (tensor-core path); other
 * shapes return MQA_ERR_UNSUPPORTED before any launch.  A length read on the
 * device that exceeds max_seqlen or runs past `total` rows is cut there and
 * MQA_FLAG_LEN_CLAMPED is set; rows outside the arrays are never touched.
 * Bounded waits report MQA_FLAG_PIPE_TIMEOUT.  Asynchronous on `stream`.
 */
MQA_API mqa_status_t mqa_prefill(void* o, const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                 int b, int total, int max_seqlen, int h, int g, int d_k, int d_v, float scale,
                                 int causal, mqa_dtype_t dtype, int32_t* status_flags, cudaStream_t stream);

/* Static, NUL-terminated name of a status code. */
MQA_API const char* mqa_status_string(mqa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* LIBMQA_MQA_H */
