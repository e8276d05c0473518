/*
 * lod.h -- C ABI of the Level-of-Detail (LoD) attention library for NVIDIA
 * B200 (sm_100a).
 *
 * The method: "Level of Detail Attention: allocating resolution instead of
 * sparsity" (featherless.ai blog), section "How It Works".  After every chunk
 * of 256 tokens the chunk's keys are clustered into groups and each group is
 * cut into pages of 16 keys; a query scores the group centroids, opens the
 * top 8 groups, scores those groups' page summaries, opens the top 2 pages of
 * each, attends exactly to the opened pages, a block-granular sliding window
 * and the sink tokens, and adds every unopened group or page as one coarse
 * entry (mean key logit + ln(count), mean value) to the SAME softmax.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer named as "device" must be CUDA device memory (or managed
 *    memory) on the current device; host pointers are marked "host".  The
 *    per-call buffers (q, out, lse, sel_groups, sel_pages, seq_lens, k_new,
 *    v_new, status) may also be page-locked host memory mapped at its host
 *    address (cudaHostAlloc / cudaMallocHost under unified addressing): the
 *    kernels then read or write those bytes over the host link themselves,
 *    with no separate copy.  Inputs in such host memory (q, k_new, v_new)
 *    must be written by the host before the call is enqueued, not by GPU
 *    work still pending on the stream: the kernels may read them as soon as
 *    they start, before earlier kernels on the stream have finished (device
 *    inputs are read only after that).  The entry points check these buffers
 *    and refuse pageable host memory and another device's memory
 *    (LOD_EINVAL) before anything is enqueued.  The KV cache, the index and
 *    the workspace must be device memory.
 *  - The caller owns every buffer.  The library never allocates or frees
 *    device memory and never synchronises the stream, with one exception:
 *    lod_get_status() copies 4 bytes to the host and waits for them.
 *  - All work is enqueued asynchronously on `stream` (NULL = legacy default
 *    stream).  Calls are reentrant; two calls that share a workspace must be
 *    ordered on the GPU (same stream, or events).
 *  - Tensors are dense, row-major, with the innermost dimension contiguous.
 *    The KV cache is addressed as K[b][h][t][:] = K + b*s[0] + h*s[1] + t*s[2]
 *    (strides in ELEMENTS, s = kv_strides); every stride and the base pointer
 *    must be 16-byte aligned.
 *  - Return value: LOD_OK, or a negative lod_status.  On failure nothing was
 *    enqueued and lod_last_error() (thread-local) describes the problem.
 *  - Index values read back from device memory (page ranges, member
 *    offsets, sequence lengths) are bounds-checked by the kernels; a bad value
 *    is skipped, never dereferenced, and recorded in a device status word that
 *    lod_get_status() returns (LOD_EDEVICE).
 */
#ifndef LOD_H_
#define LOD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lod_stream_t;

typedef enum {
  LOD_OK = 0,
  LOD_EINVAL = -1,       /* null pointer, bad shape or stride, misalignment, range */
  LOD_EUNSUPPORTED = -2, /* a valid but unimplemented configuration */
  LOD_ECUDA = -3,        /* a CUDA launch or runtime call failed */
  LOD_EDEVICE = -4       /* a kernel found and skipped a bad index value */
} lod_status;

typedef enum { LOD_DTYPE_F32 = 0, LOD_DTYPE_BF16 = 1 } lod_dtype;
typedef enum { LOD_OP_BUILD = 0, LOD_OP_DECODE = 1, LOD_OP_PREFILL = 2 } lod_op;

/* Device status bits (lod_get_status). */
#define LOD_ST_BAD_SEQLEN 0x1u   /* seq_len outside [1, Tmax]: that row's output is zeroed */
#define LOD_ST_BAD_PAGE 0x2u     /* page range or page slot outside the chunk's slots */
#define LOD_ST_BAD_MEMBER 0x4u   /* a page's member run [pBeg, pBeg + pCnt) outside the chunk */
#define LOD_ST_BAD_COUNT 0x8u    /* group or page count outside [0, chunk] */
#define LOD_ST_TIMEOUT 0x10u     /* an asynchronous copy did not complete within the kernel's wait limit */

/*
 * Parameters.  Supported: dtype F32 or BF16 (cache, summaries, q and out all
 * in this dtype); d in {64, 128}; chunk = 256 and page = 16 (the page's
 * values); 1 <= clusters <= 16; 1 <= kmeans_iters <= 64; 1 <= top_groups
 * <= 16; 0 <= top_pages <= 4 (0: two-tier LoD, an opened group is opened
 * whole with no page tier); window a positive multiple of chunk (the
 * page says 256-512); 0 <= sinks < chunk; Hq a multiple of Hkv with
 * Hq/Hkv a power of two no larger than 8; Tmax a positive multiple of chunk.
 * scale <= 0 selects 1/sqrt(d).  kv_bits 0 or 4: 4 is the pages' three-tier
 * INT4 mode ("Level of Detail Attention", the paragraph after the quality
 * tables: INT4 KV storage, only the selected pages decompressed), where the
 * members of every indexed page are kept as 4-bit codes of a per-page,
 * per-channel quantiser (see lod_index) and an opened page is read from
 * them; it needs top_pages >= 1.  The summaries, the sinks and the window
 * always use the cache dtype.  head_shard: a process that holds KV heads
 * [first, first + Hkv) of a model with more KV heads (tensor-parallel
 * attention) passes (model KV heads << 16) | first, so that the k-means
 * initialisation of sequence b, head h uses the model-wide index
 * b * (model KV heads) + first + h and the shard's index equals the one an
 * unsharded process builds; 0 for an unsharded model.
 */
typedef struct lod_params {
  int32_t dtype;        /* lod_dtype */
  int32_t B;            /* batch (sequences) */
  int32_t Hq;           /* query heads */
  int32_t Hkv;          /* KV heads; query head h reads KV head h / (Hq/Hkv) */
  int32_t d;            /* head dimension */
  int32_t chunk;        /* tokens per indexed chunk: 256 */
  int32_t page;         /* keys per page: 16 */
  int32_t clusters;     /* k-means groups per chunk */
  int32_t kmeans_iters; /* Lloyd rounds */
  int32_t top_groups;   /* groups opened per query: 8 */
  int32_t top_pages;    /* pages opened per opened group: 2; 0 = every page (two-tier LoD) */
  int32_t window;       /* sliding window in tokens (block granular) */
  int32_t sinks;        /* sink tokens at positions [0, sinks) */
  int32_t kv_bits;      /* 0: opened pages read in the cache dtype; 4: three-tier INT4 */
  uint64_t seed;        /* k-means initialisation seed */
  float scale;          /* softmax scale on q.k; <= 0 means 1/sqrt(d) */
  int32_t head_shard;   /* 0, or (model KV heads << 16) | first KV head of this shard */
  int64_t Tmax;         /* capacity of the KV cache and of the index, in tokens */
} lod_params;

/*
 * The multi-resolution index (all device pointers, caller-owned, sized by
 * lod_index_sizes).  With Cmax = Tmax / chunk, k = clusters and
 * P = chunk/page + k page slots per chunk, per (b, kvh) sequence:
 *   gK, gV  [Cmax*k][d]   group mean key / value, cache dtype (0 if empty)
 *   gCnt    [Cmax*k]      int32 group size (0 = empty group, skipped)
 *   pK, pV  [Cmax*P][d]   page mean key / value, cache dtype
 *   pCnt    [Cmax*P]      int32 page size (0 = unused slot)
 *   pBeg    [Cmax*P]      int16 first member of the page, offset into perm
 *   gPage   [Cmax*(k+1)]  int16 pages of group j are slots [gPage[j], gPage[j+1])
 *   perm    [Cmax*chunk]  int16 chunk-local token offsets, group-major and
 *                         ascending within a group; -1 past the last member
 *   mK, mV  [Cmax*chunk][d] member-ordered copies of the chunk's keys and
 *                         values: row m of chunk c is the token at offset
 *                         perm[m], so the members of a page are the
 *                         consecutive rows [pBeg, pBeg + pCnt) and an opened
 *                         page is read as one contiguous run (rows past the
 *                         last member are not written)
 *   gMeta   [Cmax*k]      int32 gCnt and gPage of a group in one word:
 *                         size | first page slot << 16 | end page slot << 24
 *   qK, qV  [Cmax*chunk][d/2] uint8, kv_bits = 4 only: the member-ordered
 *                         keys / values as 4-bit codes, two per byte
 *                         (channel 2i in the low nibble, 2i+1 in the high)
 *   qKs, qVs [Cmax*P][d][2] float, kv_bits = 4 only: per page slot and
 *                         channel the quantiser (scale, low) over the page's
 *                         members: low = min, scale = (max - low) / 15,
 *                         code = clamp(rint((x - low) / scale), 0, 15) (0 when
 *                         scale = 0); a member reads fmaf(code, scale, low)
 * With kv_bits = 4 the member copies mK, mV are unused (size 0, may be NULL);
 * with kv_bits = 0 the four INT4 arrays are unused (size 0, may be NULL).
 * Every array is laid out [B][Hkv][...] in that order.  gK, gV, pK, pV, perm,
 * mK and mV must be 16-byte aligned, gCnt, pCnt and gMeta 4-byte aligned.
 */
typedef struct lod_index {
  void* gK;
  void* gV;
  int32_t* gCnt;
  void* pK;
  void* pV;
  int32_t* pCnt;
  int16_t* pBeg;
  int16_t* gPage;
  int16_t* perm;
  void* mK;
  void* mV;
  int32_t* gMeta;
  uint8_t* qK;
  uint8_t* qV;
  float* qKs;
  float* qVs;
} lod_index;

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t lod_version(void);

/* Last error message of the calling thread ("" when none). */
const char* lod_last_error(void);

/*
 * Byte sizes of the sixteen lod_index arrays, in field order (gK, gV, gCnt,
 * pK, pV, pCnt, pBeg, gPage, perm, mK, mV, gMeta, qK, qV, qKs, qVs), written
 * to bytes[0..15] (host); an array the parameters do not use has size 0.
 * Validates `p` like every other entry point.
 */
#define LOD_INDEX_ARRAYS 16
int32_t lod_index_sizes(const lod_params* p, size_t bytes[LOD_INDEX_ARRAYS]);

/*
 * Workspace bytes needed by one call of `op` (lod_op) with parameters `p`
 * (for LOD_OP_PREFILL: per call, whatever its Tq), written to *bytes (host).
 * The workspace is caller-owned device memory, 256-byte aligned; it holds
 * the device status word and the per-split partial softmax states.  Zero it
 * once after allocation (its status word accumulates LOD_ST_* bits until
 * lod_get_status() reads and clears it); its other bytes need no clearing.
 */
int32_t lod_workspace_bytes(const lod_params* p, int32_t op, size_t* bytes);

/*
 * Online index build ("How It Works", paragraph 1): for every sequence b and
 * KV head, and for every chunk c in [chunk_begin, chunk_end), cluster the
 * chunk's keys with k-means (seeded farthest-first initialisation, then
 * kmeans_iters Lloyd rounds, squared Euclidean distance in fp32; sink
 * positions [0, sinks) of chunk 0 are never clustered), cut each group into
 * pages of `page` keys in ascending position order, and store group and page
 * mean keys, mean values (fp32 sums rounded to the cache dtype) and counts.
 *   K, V        device, cache dtype, [B][Hkv][Tmax][d] with strides kv_strides
 *   kv_strides  host, 3 strides in elements (b, h, t)
 *   index       host struct of device pointers; chunks outside the range are
 *               left untouched
 *   ws          device workspace of at least lod_workspace_bytes(LOD_OP_BUILD)
 * Errors: LOD_EINVAL if chunk_end * chunk > Tmax or the range is empty or
 * negative.
 */
int32_t lod_build_index(const lod_params* p, const void* K, const void* V,
                        const int64_t kv_strides[3], int64_t chunk_begin, int64_t chunk_end,
                        const lod_index* index, void* ws, size_t ws_bytes, lod_stream_t stream);

/*
 * Append the current token: for every sequence b, writes k_new[b][h] and
 * v_new[b][h] (device [B][Hkv][d], cache dtype, contiguous, 16-byte aligned)
 * into the cache rows K/V[b][h][seq_lens[b] - 1] (seq_lens device [B] int64;
 * a length outside [1, Tmax] skips that sequence).  One kernel for the whole
 * batch, asynchronous on `stream`; with lod_decode after it on the same
 * stream, the decode reads the new rows.
 */
int32_t lod_append_kv(const lod_params* p, void* K, void* V, const int64_t kv_strides[3],
                      const int64_t* seq_lens, const void* k_new, const void* v_new, lod_stream_t stream);

/*
 * Online index build for decode ("How It Works", paragraph 1: the index is
 * built as inference proceeds, after every chunk of 256 tokens): for every
 * sequence b whose length seq_lens[b] (device [B] int64) is a positive
 * multiple of chunk, builds the chunk that length has just completed,
 * [seq_lens[b] - chunk, seq_lens[b]), for all KV heads, exactly as
 * lod_build_index would; other sequences are left alone.  The decision is
 * taken on the device, so the call can be issued every decode step (or every
 * step of a captured graph) on a second stream, concurrently with
 * lod_decode: a chunk completed at length L is first visible to a query at
 * position >= L - chunk + window (the block window), i.e. window - chunk
 * steps later, and the build must be ordered before that decode.  ws as for
 * lod_build_index.  Same errors as lod_build_index.
 */
int32_t lod_build_ready(const lod_params* p, const void* K, const void* V,
                        const int64_t kv_strides[3], const int64_t* seq_lens, const lod_index* index,
                        void* ws, size_t ws_bytes, lod_stream_t stream);

/*
 * LoD decode ("How It Works", paragraphs 2-3): one query per sequence b at
 * position t = seq_lens[b] - 1 (the current token's K/V is already in the
 * cache).  The exact window is [chunk * max(0, t/chunk - window/chunk + 1), t],
 * the sinks are [0, min(sinks, window start)), and the visible index is the
 * complete chunks before the window start; those chunks must have been built.
 *   q          device [B][Hq][d] cache dtype
 *   seq_lens   device [B] int64, each in [1, Tmax]
 *   out        device [B][Hq][d] cache dtype
 *   lse        device [B][Hq] float log-sum-exp of the softmax (nullable)
 *   sel_groups device [B][Hq][top_groups] int32 opened global group ids
 *              (chunk*k + slot), best first, -1 padded (nullable)
 *   sel_pages  device [B][Hq][top_groups][top_pages] int32 opened page slots
 *              (chunk*P + slot), best first, -1 padded (nullable)
 *   ws         device workspace of at least lod_workspace_bytes(LOD_OP_DECODE)
 */
int32_t lod_decode(const lod_params* p, const void* q, const void* K, const void* V,
                   const int64_t kv_strides[3], const int64_t* seq_lens, const lod_index* index,
                   void* out, float* lse, int32_t* sel_groups, int32_t* sel_pages, void* ws,
                   size_t ws_bytes, lod_stream_t stream);

/*
 * Chunked causal prefill ("How It Works", paragraphs 1-3; queries that open
 * the same group are processed together, as in "Coarse Semantic Blocks for
 * Efficient Training-Free Sparse Attention", Abstract).  Queries sit at
 * positions [q_begin, q_begin + Tq) of every sequence; q_begin is a multiple
 * of chunk and the cache holds K/V for [0, q_begin + Tq).  The call first
 * builds the index of every complete chunk inside [q_begin, q_begin + Tq)
 * (chunks before q_begin must already be built), then attends every query
 * under the same rules as lod_decode.  Because a chunk becomes visible only
 * to queries at least window/chunk chunks later, building first gives the
 * same result as attending each chunk before indexing it.
 *   q          device [B][Hq][Tq][d] cache dtype
 *   out        device [B][Hq][Tq][d] cache dtype
 *   lse        device [B][Hq][Tq] float (nullable)
 *   sel_groups device [B][Hq][Tq][top_groups] int32 (nullable)
 *   sel_pages  device [B][Hq][Tq][top_groups][top_pages] int32 (nullable)
 *   index      its chunks [q_begin/chunk, (q_begin+Tq)/chunk) are written
 *   ws         device workspace of at least lod_workspace_bytes(LOD_OP_PREFILL)
 * With bf16 caches and d = 128 (and q in device memory) the rows are
 * processed in waves of query chunks, and the rows that opened the same
 * group share tensor-core tiles (the grouped prefill); the index of the
 * next wave's chunks is built on a second stream of the library (created
 * once per device) while a wave attends, and that stream is joined back to
 * `stream` before the call's work ends.  Other configurations build the
 * whole range first and then attend per query chunk.
 */
int32_t lod_prefill(const lod_params* p, const void* q, int64_t q_begin, int64_t Tq,
                    const void* K, const void* V, const int64_t kv_strides[3],
                    const lod_index* index, void* out, float* lse, int32_t* sel_groups,
                    int32_t* sel_pages, void* ws, size_t ws_bytes, lod_stream_t stream);

/*
 * Size of the scratch array built into the library for lod_decode_noalloc.
 */
#define LOD_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * lod_decode without a workspace argument, for callers that cannot allocate
 * device memory themselves: a serving engine whose memory pool owns every
 * allocation, a runtime that may not allocate while it records a CUDA graph
 * or runs a latency-critical step, or a plugin host that hands its kernels
 * only input and output buffers.  The method's pages have no counterpart of
 * this entry point: it exists only for those callers.
 *
 * Computes exactly what lod_decode computes, with the same arguments and
 * layouts, except:
 *   - no ws / ws_bytes: the scratch lives in a fixed device array of
 *     LOD_NOALLOC_SCRATCH_BYTES (8 MiB) compiled into the library.  Every GPU
 *     that loads the library holds that array until the process exits.
 *     Shapes whose scratch (lod_workspace_bytes(LOD_OP_DECODE)) exceeds it
 *     are rejected with LOD_EINVAL and a message naming both sizes; nothing
 *     is enqueued then.  (With bf16 caches and d = 128 the 128K-context
 *     decode of 4 sequences x 8 KV heads x 8 query heads per KV head needs
 *     about 0.66 MB and a 1M-context decode of one sequence with the same
 *     heads about 0.75 MB; fp32 caches or d = 64 keep every group's score
 *     and need more, e.g. about 9.6 MB for that 1M decode in fp32.)
 *   - status: nullable device pointer to a 4-byte aligned uint32_t that
 *     receives (bitwise OR) this call's LOD_ST_* bits; the caller zeroes it
 *     (a misaligned pointer is rejected with LOD_EINVAL).  When NULL the
 *     bits are recorded in the built-in array and not reported.
 * No device memory is allocated or freed by this call, by the library or by
 * any library it calls.  The first call on each device looks up that
 * device's address of the built-in array (cudaGetSymbolAddress, with that
 * device current), and so does the first call after the device's current
 * context has changed (after cudaDeviceReset, or a context switch through
 * the driver API); make those calls outside any stream capture.  All calls on one device share the one array and it keeps the
 * last call's contents: calls whose executions can overlap on the GPU
 * (different streams without ordering, or concurrent host threads) race on
 * it and produce undefined results.  Order them on one stream.
 */
int32_t lod_decode_noalloc(const lod_params* p, const void* q, const void* K, const void* V,
                           const int64_t kv_strides[3], const int64_t* seq_lens, const lod_index* index,
                           void* out, float* lse, int32_t* sel_groups, int32_t* sel_pages,
                           uint32_t* status, lod_stream_t stream);

/*
 * Read and clear the device status word kept in `ws` (the only synchronising
 * call: it waits for `stream`).  *status (host) receives the LOD_ST_* bits
 * recorded since the last read; returns LOD_EDEVICE if any bit was set.
 */
int32_t lod_get_status(void* ws, lod_stream_t stream, uint32_t* status);

#ifdef __cplusplus
}
#endif

#endif /* LOD_H_ */
