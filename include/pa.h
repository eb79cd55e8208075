/*
 * pa.h — C ABI of the paged-KV-cache attention library (libpa.so), sm_100a.
 *
 * The library implements the data-parallel hot path of PagedAttention: the
 * KV cache is cut into fixed-size blocks of BLOCK_SIZE tokens, a per-sequence
 * block table maps logical blocks to non-contiguous physical blocks, blocks
 * are handed out on demand, and parallel samples share prompt blocks through
 * reference counts with copy-on-write (vLLM launch blog, "PagedAttention"
 * section, summarised on the CSDN discovery note, item 2; agientry.com
 * overview, opening section; gitcode repo walkthrough, section 2.1).
 *
 * Conventions for every call:
 *  - Device memory and streams belong to the caller.  No call allocates or
 *    frees device memory; scratch space is passed in through pa_opts.
 *  - Device calls are asynchronous on opts->stream (NULL opts or NULL stream
 *    means the legacy default stream) on the current CUDA device; pointers
 *    must belong to that device.
 *  - Argument errors are reported before anything is launched, with no side
 *    effects.  Errors that only the device can see (a block id outside the
 *    pool, a slot outside the cache, a context longer than its block-table
 *    row, a bounded wait that gave up) set bits in a per-device status word
 *    and the offending element is skipped (see pa_get_device_status).
 *  - Tensors are described by pa_tensor: a data pointer, a dtype, a rank and
 *    per-dimension sizes and strides (in elements).  Only the layouts listed
 *    at each call are accepted.
 *
 * Physical KV layout (part of this ABI): k_cache and v_cache are each
 *   [num_blocks, num_kv_heads, block_size, head_size], contiguous, row-major,
 * so that the page of one (block, kv head) — block_size x head_size elements,
 * 4 KiB for bf16 / head_size 128 or fp32 / head_size 64 — is one contiguous
 * run that a single bulk copy moves.  The historical layout printed on the
 * pages (K split as head_size/x by x, V transposed; gitcode walkthrough,
 * section 2.1) served per-thread-group 16-byte loads on older GPUs and is not
 * used.
 *
 * Supported: block_size 16; for the cache write and decode (bf16, head_size
 * 128), (bf16, head_size 64), (fp32, head_size 64), (fp32, head_size 128),
 * and an FP8 e4m3 cache with head_size 128 and bf16 query/output
 * (pa_reshape_and_cache_fp8, pa_decode_fp8); for multi-token attention
 * (pa_prefill) bf16 with head_size 128; num_heads / num_kv_heads in
 * {1, 2, 4, 8}.  Anything else returns PA_ERR_UNSUPPORTED.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,    /* bad pointer, shape, stride, dtype or id */
  PA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (dtype/head size/group) */
  PA_ERR_OUT_OF_BLOCKS = 3,  /* allocator: free blocks exhausted, state unchanged */
  PA_ERR_CUDA = 4,           /* a CUDA runtime call failed */
  PA_ERR_DEVICE_TIMEOUT = 5, /* a device-side bounded wait gave up */
  PA_ERR_DEVICE_BOUNDS = 6,  /* a device-side index check failed; element skipped */
  PA_ERR_SCRATCH_LIMIT = 7,  /* pa_decode_no_alloc: the call needs more scratch than the library's fixed buffer */
  PA_ERR_HOST_ALLOC = 8      /* allocator: host memory ran out inside the call (see the allocator rules) */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_I32 = 2, PA_I64 = 3, PA_FP8_E4M3 = 4 } pa_dtype;

/* A strided view of caller-owned memory.  Strides are in elements. */
typedef struct {
  void* data;
  int32_t dtype; /* pa_dtype */
  int32_t ndim;  /* 1..5 */
  int64_t shape[5];
  int64_t stride[5];
} pa_tensor;

/* Decode workspace header: the first PA_DECODE_WS_HEADER_BYTES of every
 * workspace hold the balanced split's merge counters (one 32-bit counter per
 * worker, at most PA_DECODE_WS_HEADER_BYTES / 4 workers).  They must be zero
 * before a workspace is first used; every call leaves them zero again, in
 * every split mode, including a call that times out, so a workspace
 * zero-filled once (cudaMemset, torch.zeros) serves any sequence of calls. */
#define PA_DECODE_WS_HEADER_BYTES (64u * 1024u)

typedef struct {
  void* stream;             /* cudaStream_t, NULL = legacy default stream */
  void* workspace;          /* device scratch for split decode, 256-byte aligned, may be NULL; zero-filled
                               once before its first use (see PA_DECODE_WS_HEADER_BYTES); calls whose
                               kernels may overlap on the GPU must not share it */
  size_t workspace_bytes;   /* size of workspace */
  int32_t partition_tokens; /* pa_decode context split:
                                 0  = auto: balanced split over all SMs when the
                                      workspace is large enough, else no split;
                                 >0 = fixed partitions of this many tokens (a
                                      multiple of block_size), one partial result
                                      per partition, then a log-sum-exp merge;
                                 -1 = no split: each (sequence, kv head) is
                                      reduced by one warp, no workspace needed */
  int32_t timeout_ms;       /* bound on every device-side wait; 0 = 1000 ms */
} pa_opts;
/* pa_opts departs from the survey's sketch of this struct in two fields:
 * there is no force_split (a caller forces a split by choosing
 * partition_tokens > 0, and the auto mode already splits whenever the
 * workspace allows), and timeout_ms is added, because every device-side wait
 * of this library is bounded and a caller may want a bound other than 1 s. */

/* Device status bits (pa_get_device_status). */
#define PA_DEV_TIMEOUT 0x1u     /* a bounded wait gave up */
#define PA_DEV_BAD_BLOCK 0x2u   /* block-table entry or copy pair outside [0, num_blocks) */
#define PA_DEV_BAD_CONTEXT 0x4u /* context_len < 0 or > block-table row capacity; pa_prefill: a query range that does not fit */
#define PA_DEV_BAD_SLOT 0x8u    /* slot_mapping entry < -1 or >= num_blocks*block_size */
#define PA_DEV_BAD_WORKSPACE 0x10u /* pa_decode: a merge counter of the workspace did not start at zero */

/* ---------------------------------------------------------------------------
 * Cache write (the step that stores each new token's K/V at its slot).
 * The pages imply it — tokens land in the block the table names, at their
 * offset (launch blog "PagedAttention" section; CSDN note item 2) — without
 * naming it.
 *
 *   for t, h:  s = slot_mapping[t];  if s == -1: skip
 *              k_cache[s / block_size, h, s % block_size, :] = key[t, h, :]
 *              v_cache[s / block_size, h, s % block_size, :] = value[t, h, :]
 *
 * key, value:   [T, num_kv_heads, head_size], dtype of the cache, last dim
 *               contiguous, token/head strides multiples of 16 bytes, data
 *               16-byte aligned.  T may be 0 (nothing is launched).
 * k_cache, v_cache: [num_blocks, num_kv_heads, block_size, head_size],
 *               contiguous, 16-byte aligned.
 * slot_mapping: [T] int64, contiguous.  Entries outside [-1, num_blocks*bs)
 *               set PA_DEV_BAD_SLOT and are skipped.
 * Bit copy: the cache receives the exact input bits.  Two tokens with the same
 * slot in one call race (undefined which one lands).
 * ------------------------------------------------------------------------- */
pa_status pa_reshape_and_cache(const pa_tensor* key, const pa_tensor* value, pa_tensor* k_cache,
                               pa_tensor* v_cache, const pa_tensor* slot_mapping, const pa_opts* opts);

/* ---------------------------------------------------------------------------
 * Copy-on-write block copy (launch blog "PagedAttention" section; CSDN note
 * item 2: a write into a block shared by several samples first copies it).
 *
 *   for each pair (src, dst):  k_cache[dst] = k_cache[src];  v_cache[dst] = v_cache[src]
 *   (whole block: every head, every offset)
 *
 * pairs: [n, 2] int64 in DEVICE memory, contiguous (the allocator's
 *        copy-on-write output, uploaded by the caller on the same stream).
 *        n may be 0.  A pair with an id outside [0, num_blocks) sets
 *        PA_DEV_BAD_BLOCK and is skipped.  Destinations must be distinct and
 *        no destination may be another pair's source (the allocator never
 *        emits such pairs).
 * ------------------------------------------------------------------------- */
pa_status pa_copy_blocks(pa_tensor* k_cache, pa_tensor* v_cache, const pa_tensor* pairs, const pa_opts* opts);

/* ---------------------------------------------------------------------------
 * Swap copy between a device pool and a pinned host pool (either direction):
 *   for each pair (src, dst): dst_k[dst] = src_k[src]; dst_v[dst] = src_v[src]
 * src_k/src_v and dst_k/dst_v: caches of the same dtype and [*, H_kv, 16, D]
 * shape (block counts may differ), each in device memory of the current
 * device or in page-locked host memory the device can address (e.g.
 * cudaHostAlloc, torch pin_memory); anything else is PA_ERR_INVALID_ARG.
 * pairs: [n, 2] int64 in device or pinned memory (the allocator's swap pairs).
 * Ids outside their pool set PA_DEV_BAD_BLOCK and are skipped.  One kernel
 * moves every pair; the host side of the copy crosses the host link.
 * ------------------------------------------------------------------------- */
pa_status pa_swap_blocks(const pa_tensor* src_k, const pa_tensor* src_v, pa_tensor* dst_k, pa_tensor* dst_v,
                         const pa_tensor* pairs, const pa_opts* opts);

/* ---------------------------------------------------------------------------
 * Paged decode attention (gitcode walkthrough, section 2.1: the query-key dot
 * product, softmax normalisation and weighted sum of V over K/V gathered
 * block by block; launch blog "PagedAttention" section).
 *
 *   for sequence i < B, query head h < H, with g = h / (H / num_kv_heads):
 *     s_t = scale * <query[i,h,:], K_i[t, g, :]>,  t < context_lens[i]
 *     out[i,h,:] = sum_t softmax(s)_t V_i[t, g, :]
 *   where K_i[t] = k_cache[block_tables[i][t / bs], g, t % bs, :] (same for V).
 *   context_lens[i] == 0 gives a zero row.
 *
 * out:          [B, H, head_size], cache dtype, last dim contiguous, strides
 *               multiples of 16 bytes, 16-byte aligned.  Written, never read.
 * query:        [B, H, head_size], cache dtype, same layout rules.
 * k_cache, v_cache: see the physical layout above.
 * block_tables: [B, max_blocks_per_seq] int32, last dim contiguous.  Only the
 *               first ceil(context_lens[i] / bs) entries of row i are read;
 *               each must be in [0, num_blocks) (else PA_DEV_BAD_BLOCK and the
 *               page is replaced by block 0).
 * context_lens: [B] int32.  Values above max_blocks_per_seq * bs, or below 0,
 *               set PA_DEV_BAD_CONTEXT and are clamped.
 * scale:        softmax scale (usually 1/sqrt(head_size)).
 * num_kv_heads: must equal k_cache's second dimension and divide H.
 * Accumulation is fp32; the output is rounded to the cache dtype (bf16:
 * round-to-nearest-even).  Split modes (opts->partition_tokens) change only
 * fp32 rounding order.  Fixed-partition mode leaves its per-partition
 * results in the workspace after the header: at byte offset
 * PA_DECODE_WS_HEADER_BYTES, float o[B][H][P][head_size] (normalised), then,
 * at the next multiple of 256 bytes, float lse[B][H][P] (natural log of the
 * partition's softmax denominator plus its max logit),
 * P = ceil(max_blocks_per_seq*bs / partition_tokens); entries of partitions
 * past a sequence's end are left unwritten.  The balanced split (auto mode)
 * merges the shares of a row cut between workers inside the same launch:
 * the worker whose pages complete the row merges it, so no worker waits for
 * another and no assumption is made about which CTAs run at the same time.
 * B may be 0.  B must be < 2^20.
 * ------------------------------------------------------------------------- */
pa_status pa_decode(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                    const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                    int32_t num_kv_heads, const pa_opts* opts);

/* Launch shape of pa_decode on the current process (a tuning knob; 0 keeps
 * the default): warps per CTA (each warp is one worker with its own page
 * ring; G = num_heads / num_kv_heads.  bf16 or fp32 cache: default 8 for
 * G = 1 or 8 and 12 for G = 2 or 4, at most 12 (8 for bf16 at G = 8).  FP8
 * cache: default and most 16 up to G = 4, 8 at G = 8), ring stages per warp
 * (default 2; lowered automatically to fit shared memory), CTAs per SM
 * (default 1).  Changes the workspace size of the auto mode.  Not
 * thread-safe. */
pa_status pa_set_decode_tuning(int32_t warps_per_cta, int32_t stages, int32_t ctas_per_sm);

/* ---------------------------------------------------------------------------
 * pa_decode without a caller workspace.  The pages have no counterpart to
 * this call; it exists for callers that cannot provide device scratch: for
 * instance code running inside a host framework that owns every device
 * allocation and passes plugins no scratch buffer, or a serving loop that
 * must not call cudaMalloc (which can synchronise the device and stall other
 * streams).  It computes exactly what pa_decode computes, with the same
 * arguments and split modes (opts->partition_tokens, stream, timeout_ms;
 * opts->workspace and workspace_bytes are ignored), but its split-context
 * scratch is a fixed array of PA_NO_ALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.
 *  - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *    routine.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - A call whose split needs more scratch than PA_NO_ALLOC_SCRATCH_BYTES
 *    returns PA_ERR_SCRATCH_LIMIT before launching anything (use
 *    partition_tokens -1, no split, which needs none).
 *  - In the auto mode (partition_tokens 0) a split that needs more than the
 *    array holds (e.g. after pa_set_decode_tuning raised the worker count)
 *    runs unsplit, as pa_decode does when its workspace is too small.
 *  - All calls share the array and it keeps the last call's contents.  Its
 *    header of merge counters is zero when the library is loaded and every
 *    call leaves it zero; every other byte a call reads was written earlier
 *    in that same call.  Calls whose kernels overlap on the GPU (two
 *    streams, or two host threads) race on it: issue them on one stream.
 * ------------------------------------------------------------------------- */
#define PA_NO_ALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
pa_status pa_decode_no_alloc(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                             const pa_tensor* v_cache, const pa_tensor* block_tables,
                             const pa_tensor* context_lens, float scale, int32_t num_kv_heads, const pa_opts* opts);

/* ---------------------------------------------------------------------------
 * Shared-prefix decode.  The pages state that reference counts and
 * copy-on-write let parallel samples of one prompt share the prompt's memory
 * and its computation (CSDN discovery note, item 2, on the vLLM launch
 * blog's "PagedAttention" section).  pa_decode shares the memory only: each
 * sample still reads every prompt block.  This call also shares the reads:
 * the batch is cut into groups of consecutive sequences whose block tables
 * begin with the same group_blocks[v] blocks; one kernel row per (group, kv
 * head) carries the query heads of every member, attends the shared pages
 * with all of them (each shared page is read once for the whole group), then
 * each member's own remaining pages with that member's heads only.  The
 * output is pa_decode's (the same formula; only fp32 rounding order
 * differs).  One kernel launch.
 *
 * group_start:  [n_groups + 1] int32 on the device: group v holds sequences
 *               group_start[v] .. group_start[v+1] - 1; group_start[0] = 0,
 *               non-decreasing, group_start[n_groups] = B, at most
 *               max_group_size members each (else PA_DEV_BAD_CONTEXT and
 *               every sequence is decoded on its own: the output stays
 *               right).
 * group_blocks: [n_groups] int32 on the device: leading blocks every member
 *               of the group holds (the same block ids at the same table
 *               indices; not checked).  Values above a member's number of
 *               full blocks are capped (PA_DEV_BAD_CONTEXT).  0 = no
 *               sharing.  pa_alloc_prefix_groups computes both from the
 *               allocator.
 * max_group_size: most members a group may have; (num_heads / num_kv_heads)
 *               * max_group_size must be 1, 2, 4 or 8 (else
 *               PA_ERR_UNSUPPORTED).
 * Other arguments as pa_decode; bf16 with head_size 128 or fp32 with
 * head_size 64.  opts->partition_tokens: 0 (balanced split: needs a
 * workspace of pa_decode_cascade_workspace_bytes, zero-filled before first
 * use, as for pa_decode) or -1 (no split, no workspace); fixed partitions
 * are PA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_cascade(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                            const pa_tensor* v_cache, const pa_tensor* block_tables, const pa_tensor* context_lens,
                            const pa_tensor* group_start, const pa_tensor* group_blocks, int32_t max_group_size,
                            float scale, int32_t num_kv_heads, const pa_opts* opts);
/* Workspace bytes of pa_decode_cascade for these sizes on the current
 * device (partition_tokens 0; 0 bytes for -1). */
pa_status pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                            int32_t head_size, int32_t max_group_size, int32_t partition_tokens,
                                            size_t* bytes_out);

/* ---------------------------------------------------------------------------
 * FP8 (e4m3) KV cache.  The pages say only that the KV cache itself can be
 * quantized to save memory (gitcode walkthrough, section 三 "量化", the
 * quantized_kvcache item); this library's form: every K (V) element is stored
 * as one OCP e4m3 code of value / k_scale[h] (v_scale[h]), h the kv head,
 * so a page is 2 KiB at head_size 128 and the decode reads half the bytes.
 *
 * pa_reshape_and_cache_fp8: as pa_reshape_and_cache, with key/value bf16 or
 *   fp32 and k_cache/v_cache of dtype PA_FP8_E4M3 [num_blocks, H_kv, 16, 128];
 *   code = e4m3(float(x) / scale[h]) with IEEE fp32 division, rounding to
 *   nearest even and saturation to +-448 (NaN stays NaN).
 * pa_decode_fp8: as pa_decode over an FP8 cache with bf16 query and output;
 *   K[t] = e4m3_value(code) * k_scale[g], V likewise; fp32 accumulation.
 *   For G = H / H_kv >= 2 the page dot products run on the tensor cores
 *   (mma.sync, f16 operands): the e4m3 codes are exact in f16 and the
 *   query, scaled per head by a power of two, is carried as an f16 high
 *   part plus the f16 rounding of the rest (about 22 bits), so the logits
 *   keep close to fp32 accuracy at any query magnitude; the probabilities
 *   enter the PV product as f16.
 * k_scale, v_scale: [H_kv] fp32 on the device, contiguous, positive.
 * pa_reshape_and_cache and pa_decode reject FP8 caches (they have no scales).
 * ------------------------------------------------------------------------- */
pa_status pa_reshape_and_cache_fp8(const pa_tensor* key, const pa_tensor* value, pa_tensor* k_cache,
                                   pa_tensor* v_cache, const pa_tensor* slot_mapping, const pa_tensor* k_scale,
                                   const pa_tensor* v_scale, const pa_opts* opts);
pa_status pa_decode_fp8(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                        const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                        int32_t num_kv_heads, const pa_tensor* k_scale, const pa_tensor* v_scale,
                        const pa_opts* opts);

/* ---------------------------------------------------------------------------
 * Multi-token (chunked-prefill) paged attention.  The pages list chunked
 * prefill among the serving-loop optimisations: a long prompt's prefill is
 * cut into chunks that run in the same step as decode requests (gitcode
 * walkthrough, section 2.2); the attention is the section 2.1 computation
 * applied to every new token, causally:
 *
 *   sequence i has n_i = query_start[i+1] - query_start[i] new tokens at
 *   positions c_i + j (c_i = context_lens[i] - n_i; their K/V must already
 *   be in the cache, e.g. by pa_reshape_and_cache earlier on the stream);
 *   for row r = query_start[i] + j and query head h, g = h / (H / H_kv):
 *     s_t = scale * <query[r,h,:], K_i[t, g, :]>,  t = 0 .. c_i + j
 *     out[r,h,:] = sum_t softmax(s)_t V_i[t, g, :]
 *
 * A decode request is n_i = 1; a whole prompt is n_i = context_lens[i];
 * n_i = 0 writes nothing.  Runs on the tensor cores (tcgen05): QK^T and PV
 * in bf16 with fp32 accumulation; the softmax is fp32 (its denominator summed
 * before rounding), the probabilities are rounded to bf16 for the PV
 * product, and the output is rounded to nearest even.
 *
 * out, query:   [T, H, 128] bf16, last dim contiguous, strides multiples of
 *               16 bytes, 16-byte aligned (T = total new tokens).  Rows not
 *               covered by any sequence are left unwritten.
 * k_cache, v_cache: bf16 [num_blocks, H_kv, 16, 128] (layout above).
 * block_tables: [B, max_blocks_per_seq] int32 (entries past
 *               ceil(context_lens[i] / 16) are not read; bad ids set
 *               PA_DEV_BAD_BLOCK and are replaced by block 0).
 * context_lens: [B] int32, tokens of sequence i after the step.
 * query_start:  [B + 1] int32 on the device, non-decreasing, query_start[0]
 *               >= 0, query_start[B] <= T.  A sequence with n_i < 0,
 *               n_i > context_lens[i], rows outside [0, T), context_lens[i]
 *               above the table capacity, or n_i > max_query_len sets
 *               PA_DEV_BAD_CONTEXT and is skipped.
 * max_query_len: host-side bound on every n_i (sizes the grid).
 * scale:        softmax scale, finite and > 0.
 * H / H_kv in {1, 2, 4, 8}; B <= 65535.  No workspace.  Other dtypes or
 * head sizes return PA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------- */
pa_status pa_prefill(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                     const pa_tensor* block_tables, const pa_tensor* context_lens, const pa_tensor* query_start,
                     int32_t max_query_len, float scale, int32_t num_kv_heads, const pa_opts* opts);

/* Workspace bytes pa_decode needs on the current device for these sizes and
 * this partition_tokens setting (0 = auto/balanced, >0 = fixed, -1 = none),
 * header included; 0 for -1.  Departs from the survey's sketch
 * (num_seqs, num_heads, head_size, max_context_len, partition_tokens) ->
 * size_t: it takes num_kv_heads, because the balanced split's shares hold
 * one row per query head of a kv-head group, and max_blocks_per_seq (the
 * block-table width the decode call will get) instead of a token count, and
 * it returns a status with the size in *bytes_out, so that bad arguments and
 * a missing device are reported rather than folded into a size.  The auto
 * mode's size depends on the current device's SM count and on
 * pa_set_decode_tuning: it is per device, so size a workspace on the device
 * that will run the decode. */
pa_status pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                    int32_t head_size, int32_t max_blocks_per_seq, int32_t partition_tokens,
                                    size_t* bytes_out);

/* ---------------------------------------------------------------------------
 * Host block allocator (launch blog "PagedAttention" section; CSDN note item
 * 2; agientry.com overview).  Pure host code, not thread-safe (the caller
 * serialises), no CUDA needed.
 *
 * Rules (the pages give the mechanism; the orders are this library's):
 *  - free blocks form a LIFO stack seeded from free_order (free_order[0] is
 *    handed out first; NULL = 0, 1, 2, ...); a freed block goes on top;
 *  - appending token at position p: if p % bs == 0 a fresh block is taken;
 *    otherwise, if the last block's reference count is above 1, a fresh block
 *    is taken, the pair (old, new) is reported for pa_copy_blocks, the old
 *    block loses one reference and the table points at the new block
 *    (copy-on-write; at most one pair per append call); the token's slot is
 *    table[p / bs] * bs + p % bs;
 *  - an append is all-or-nothing: PA_ERR_OUT_OF_BLOCKS leaves every state
 *    unchanged;
 *  - fork: the child gets a copy of the parent's table and length; each block
 *    gains one reference;
 *  - free: blocks lose one reference in table order; a block reaching 0 is
 *    pushed on the free stack.
 * Sequence ids are arbitrary int64 values.  No C++ exception leaves these
 * calls: if host memory runs out inside one, it returns PA_ERR_HOST_ALLOC
 * (pa_alloc_create then creates nothing; after any other call the
 * allocator's state is unspecified and it should only be destroyed).
 * ------------------------------------------------------------------------- */
typedef struct pa_allocator pa_allocator;

typedef struct {
  int32_t num_blocks;
  int32_t num_free;      /* blocks available to allocation: free + evictable */
  int32_t num_seqs;
  int32_t block_size;
  int64_t num_tokens;    /* sum of sequence lengths (shared tokens counted per sequence) */
  int64_t waste_slots;   /* unused slots of blocks in use (bs minus the most any holder filled) */
  int32_t num_cached;    /* registered prefix-cache blocks (held or evictable) */
  int32_t num_evictable; /* registered blocks nobody holds */
} pa_alloc_stats;

/* A new allocator over blocks 0 .. num_blocks-1 of block_size tokens (both
 * > 0).  free_order: NULL, or a permutation of 0 .. num_blocks-1 (anything
 * else is PA_ERR_INVALID_ARG).  *out is the caller's, released with
 * pa_alloc_destroy (NULL is a no-op); on any error (out not NULL) *out is
 * NULL. */
pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order, pa_allocator** out);
void pa_alloc_destroy(pa_allocator* a);
/* A new empty sequence; an id already present is PA_ERR_INVALID_ARG. */
pa_status pa_seq_add(pa_allocator* a, int64_t seq_id);
/* Appends n_tokens (>= 0) tokens with unknown ids.  slots_out: [n_tokens]
 * (may be NULL when n_tokens == 0); cow_pair_out: [2] (nullable), written
 * (src, dst) when *n_cow_out (nullable) is 1.  An unknown or swapped-out
 * sequence, or a length past INT32_MAX, is PA_ERR_INVALID_ARG. */
pa_status pa_seq_append(pa_allocator* a, int64_t seq_id, int32_t n_tokens, int64_t* slots_out,
                        int64_t* cow_pair_out, int32_t* n_cow_out);
/* Appends n_tokens[k] tokens to seq_ids[k] for k = 0..n-1 in order.  Each
 * sequence's append is all-or-nothing; the call stops at the first failure and
 * *n_done_out says how many sequences were served.  slots_out holds the slots
 * of the served sequences back to back; cow_pairs_out [n, 2] holds the
 * *n_cow_out copy pairs in order. */
pa_status pa_seq_append_batch(pa_allocator* a, const int64_t* seq_ids, const int32_t* n_tokens, int32_t n,
                              int64_t* slots_out, int64_t* cow_pairs_out, int32_t* n_cow_out, int32_t* n_done_out);
/* child (a new id) starts as a copy of parent (present, not swapped out):
 * same table and length, one more reference on each block. */
pa_status pa_seq_fork(pa_allocator* a, int64_t parent, int64_t child);

/* Prefix caching.  The pages give the effect — requests reuse the computed
 * KV of an identical prefix such as a system prompt (gitcode walkthrough,
 * section 2.2, "Prefix caching (APC)"); blocks can be shared across requests
 * (agientry.com overview, opening section) — and this is the mechanism:
 *  - a sequence whose token ids are all known (created by pa_seq_add or
 *    pa_seq_add_prefix and extended only by pa_seq_append_tokens) registers
 *    each block when it becomes full, under the key (previous block of the
 *    sequence or -1, the block's token ids), if that previous block is
 *    registered (or it is the first block) and the key is not taken; so a key
 *    match means the whole prefix matches, exactly (no hashing shortcut);
 *  - pa_seq_add_prefix(seq, tokens, n) creates the sequence on the longest
 *    chain of registered keys along tokens, at most (n - 1) / bs blocks so
 *    one token is left to compute; *n_cached_out = tokens reused (a multiple
 *    of bs).  The caller then appends tokens[*n_cached_out:] with
 *    pa_seq_append_tokens and writes only their K/V;
 *  - a registered block whose count drops to 0 becomes evictable (kept in
 *    least-recently-freed order) instead of free; allocation takes the free
 *    stack first, then evicts the least recently freed evictable block;
 *    unregistering a block (eviction) unregisters its registered children in
 *    increasing block order, depth first, and frees those nobody holds;
 *  - pa_seq_append (token ids unknown) turns a sequence's registration off.
 * Without these calls the allocator behaves exactly as described above. */
pa_status pa_seq_add_prefix(pa_allocator* a, int64_t seq_id, const int64_t* tokens, int32_t n_tokens,
                            int32_t* n_cached_out);
pa_status pa_seq_append_tokens(pa_allocator* a, int64_t seq_id, const int64_t* tokens, int32_t n_tokens,
                               int64_t* slots_out, int64_t* cow_pair_out, int32_t* n_cow_out);
/* Evictable blocks, least recently freed first. */
pa_status pa_alloc_evictable(const pa_allocator* a, int32_t* out, int32_t cap, int32_t* n_out);

/* Swapping.  The pages say blocks can be swapped out (agientry.com overview,
 * opening section); this library's form:
 *  - pa_alloc_set_host_pool gives the allocator num_host_blocks host blocks
 *    (LIFO, host_free_order[0] first; NULL = 0, 1, ...); not while any
 *    sequence is swapped out;
 *  - pa_seq_swap_out gives each block of the sequence, in table order, a host
 *    block (all or nothing: PA_ERR_OUT_OF_BLOCKS), writes (device, host) pairs
 *    to pairs_out [n, 2] (cap pairs of room), then releases the device blocks
 *    as pa_seq_free would; shared blocks are copied and keep their holders;
 *  - pa_seq_swap_in takes device blocks for the host blocks in order (all or
 *    nothing), writes (host, device) pairs, returns the host blocks, and
 *    re-registers the full blocks for prefix reuse when the token ids are
 *    known;
 *  - a swapped-out sequence accepts only pa_seq_swap_in and pa_seq_free;
 *  - the caller moves the bytes with pa_swap_blocks (out: before any device
 *    block it released is written again; in: before the sequence is read). */
pa_status pa_alloc_set_host_pool(pa_allocator* a, int32_t num_host_blocks, const int32_t* host_free_order);
pa_status pa_seq_swap_out(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int32_t cap, int32_t* n_out);
pa_status pa_seq_swap_in(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int32_t cap, int32_t* n_out);
int32_t pa_alloc_num_host_free(const pa_allocator* a);
/* Host blocks of a swapped-out sequence, in table order (else
 * PA_ERR_INVALID_ARG). */
pa_status pa_seq_host_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out);
/* Releases the sequence's blocks (device, or host if swapped out) and
 * forgets the id; an unknown id (e.g. a second free) is PA_ERR_INVALID_ARG. */
pa_status pa_seq_free(pa_allocator* a, int64_t seq_id);
pa_status pa_seq_len(const pa_allocator* a, int64_t seq_id, int32_t* len_out);
/* The sequence's block table.  For a known sequence *n_out is set to the
 * table's length; if that exceeds cap the call is PA_ERR_INVALID_ARG and out
 * is not written (the same holds for the other out/cap/n_out calls, so a
 * caller can size its buffer from *n_out and call again). */
pa_status pa_seq_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out);
/* Fills out [n, max_blocks] (row-major) with the tables of seq_ids, padding
 * with -1, and context_lens_out [n] (nullable) with their lengths.  A table
 * longer than max_blocks is PA_ERR_INVALID_ARG (nothing written). */
pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int32_t n, int32_t* out,
                                int32_t max_blocks, int32_t* context_lens_out);
/* Groups for pa_decode_cascade: cuts the batch seq_ids[0..n) (in that
 * order) into runs of consecutive sequences that share their leading blocks
 * (forks of one prompt, placed next to each other).  Greedy: a run starts at
 * a sequence with its full blocks as the shared count; the next sequence
 * joins while the run has fewer than max_group_size members, the two tables
 * begin with at least one common full block, and joining keeps at least half
 * of the run's shared count (which becomes the common count).  A run of one
 * sequence gets 0 shared blocks.  Writes group_start_out [n_groups + 1]
 * (first member of each run, then n), group_blocks_out [n_groups] (shared
 * full blocks, each a block every member's table holds at the same index)
 * and *n_groups_out (<= n).  An unknown or swapped-out id is
 * PA_ERR_INVALID_ARG.  The grouping affects only speed: any grouping whose
 * members really share their first group_blocks blocks decodes to the same
 * result. */
pa_status pa_alloc_prefix_groups(const pa_allocator* a, const int64_t* seq_ids, int32_t n, int32_t max_group_size,
                                 int32_t* group_start_out, int32_t* group_blocks_out, int32_t* n_groups_out);
/* Blocks available to allocation (free plus evictable); -1 for NULL. */
int32_t pa_alloc_num_free(const pa_allocator* a);
int32_t pa_block_refcount(const pa_allocator* a, int32_t block); /* -1 if out of range */
pa_status pa_alloc_get_stats(const pa_allocator* a, pa_alloc_stats* out);

/* ---------------------------------------------------------------------------
 * Device status and diagnostics
 * ------------------------------------------------------------------------- */
/* Synchronises opts->stream, then reads and clears the current device's
 * status word into *bits_out (nullable).  Returns PA_ERR_DEVICE_TIMEOUT if the
 * timeout bit was set, else PA_ERR_DEVICE_BOUNDS if any other bit was set,
 * else PA_OK.  Departs from the survey's sketch (opts only) by the bits_out
 * out-parameter, so a caller can tell which check fired. */
pa_status pa_get_device_status(const pa_opts* opts, uint32_t* bits_out);

/* Launches one warp that waits, with the same bounded wait the decode
 * pipeline uses, on a barrier nothing completes.  It must give up after
 * opts->timeout_ms and set PA_DEV_TIMEOUT; the context stays usable.  No copy
 * is in flight during the wait. */
pa_status pa_debug_wait_selftest(const pa_opts* opts);

const char* pa_status_string(pa_status s);

/* Library version, for the Python loader's sanity check. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
