/*
 * pa.h: C ABI of libpa.so, paged-KV attention on NVIDIA B200 (sm_100a).
 *
 * The method. The KV cache is split into fixed-size blocks of 16 tokens that
 * live anywhere in one physical pool. Each sequence keeps a table that maps
 * its logical blocks to physical ones. Attention reads K/V block by block
 * through that table ("vLLM and PagedAttention", ai.zenoagi.com, §2 "The
 * PagedAttention Solution" and "Reworking the Attention Computation";
 * "vLLM — PagedAttention and Continuous Batching", s-samarth.github.io, §2.2
 * and §2.4). A sequence takes a new block only when its last one is full, so
 * only the last block can be partly filled ("How vLLM Works?",
 * peterindia.net, §03).
 *
 * Conventions for every call:
 *  - All tensor pointers are caller-owned DEVICE memory on the current CUDA
 *    device. They are row-major and contiguous, and 16-byte aligned. The
 *    library allocates nothing and keeps no state except a cached SM count
 *    per device and one device status word (pa_get_status).
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream. Calls only enqueue work, never synchronize (except
 *    pa_get_status) and never allocate, so they can be captured in CUDA graphs.
 *  - Element type of q, k, v, the caches and out is shape->dtype. The
 *    tables, lengths and slot mapping are int32/int64 as declared.
 *  - Return value: PA_OK, or a negative pa_error. On an argument error
 *    nothing is launched. PA_ERR_CUDA means a launch failed; the CUDA error
 *    stays readable with cudaGetLastError().
 *  - Bad data inside device buffers cannot be checked on the host without a
 *    sync: a table entry outside the pool, a slot outside the pool, a
 *    context length over the table's capacity. The kernels check these as
 *    they read them. A bad item is skipped (never dereferenced) and a flag is
 *    set in the device status word (PA_STATUS_*). Outputs that depended on
 *    it are then unspecified. Read the word with pa_get_status().
 *
 * Layouts (B = sequences, H = query heads, Hk = KV heads, D = head_dim,
 * NB = pool blocks, S = block size = 16, MB = table width):
 *   k_cache, v_cache : [NB][S][Hk][D]   (the kernel sketch's
 *                      [num_blocks, block_size, num_heads, d_head] comment
 *                      in "vLLM and PagedAttention" §2, with KV heads)
 *   block_tables     : int32 [B][MB], physical block of logical block i
 *   context_lens     : int32 [B], tokens in the sequence INCLUDING this
 *                      step's new ones (the cache write comes first)
 *   q, out           : [tokens][H][D]. The sketch's output comment
 *                      "[seq_len, d_model]" is read as this.
 *   k, v (new tokens): [T][Hk][D]
 * Query head h uses KV head h / (H / Hk) (contiguous groups).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 7
#define PA_BLOCK_SIZE 16

typedef enum {
    PA_DTYPE_F32 = 0,  /* IEEE fp32 */
    PA_DTYPE_BF16 = 1, /* bfloat16 */
} pa_dtype;

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARGUMENT = -1, /* null pointer, negative size, inconsistent sizes */
    PA_ERR_UNSUPPORTED = -2,      /* shape/dtype combination not compiled in */
    PA_ERR_ALIGNMENT = -3,        /* a pointer is not 16-byte aligned */
    PA_ERR_WORKSPACE = -4,        /* workspace missing or smaller than pa_decode_workspace_bytes */
    PA_ERR_CUDA = -5,             /* a CUDA runtime call or launch failed */
    PA_ERR_DEVICE = -6,           /* no usable device, or not an sm_100 device */
    PA_ERR_SCRATCH_LIMIT = -7,    /* pa_decode_noalloc: request larger than its built-in scratch */
} pa_error;

/* Flags of the device status word (OR-ed together). */
#define PA_STATUS_BAD_BLOCK_ID 0x1u   /* table entry outside [0, NB) */
#define PA_STATUS_BAD_SLOT 0x2u       /* slot_mapping entry >= NB * 16 */
#define PA_STATUS_BAD_CONTEXT 0x4u    /* context length < 0, > MB * 16, or > max_context_len */
#define PA_STATUS_WAIT_TIMEOUT 0x8u   /* a bounded wait on an async copy gave up */
#define PA_STATUS_BAD_QUERY 0x10u     /* prefill: q_len > context_len or cu_q_lens not increasing */

typedef struct {
    int32_t num_heads;    /* H, query heads */
    int32_t num_kv_heads; /* Hk, KV heads; H % Hk == 0 and H / Hk in {1, 2, 4, 8} */
    int32_t head_dim;     /* D: 64 or 128 */
    int32_t block_size;   /* tokens per block: must be 16 */
    int64_t num_blocks;   /* NB, blocks in the pool */
    int32_t dtype;        /* pa_dtype of q, out and the new tokens' k, v */
    /*
     * 0: the caches hold `dtype`. 1: they hold FP8 E4M3 codes, one byte per
     * element (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
     * infinities, largest finite 448). A cached value means code * k_scale
     * (keys) or code * v_scale (values). The write quantizes
     * fp32(x) * fp32(1 / scale) to the nearest code (ties to even, saturating
     * at +-448). FP8 caches need dtype = PA_DTYPE_BF16. The pages name FP8
     * only for weights ("vLLM and PagedAttention" §5); an FP8 cache halves the
     * bytes decode reads.
     */
    int32_t kv_fp8;
    float k_scale; /* > 0 when kv_fp8; ignored otherwise */
    float v_scale; /* > 0 when kv_fp8; ignored otherwise */
} pa_shape;

/*
 * pa_reshape_and_cache: append this step's new tokens to the cache.
 *
 * For every t in [0, num_tokens) with slot_mapping[t] >= 0, copy the [Hk][D]
 * row k[t] to k_cache viewed as [NB*16][Hk][D] at row slot_mapping[t], and
 * the same for v. A slot is physical_block * 16 + row. A negative slot means
 * padding and that token is skipped. Every other byte of the caches is left
 * alone and the copy is bit-exact. This is the on-demand slot fill of
 * "vLLM and PagedAttention" §2 "The PagedAttention Solution" ("the 7th block
 * is only requested when the 100th token is generated") and of
 * "How vLLM Works?" §03.
 *
 *   k, v         : [num_tokens][Hk][D] device
 *   k_cache,
 *   v_cache      : [NB][16][Hk][D] device, updated in place
 *   slot_mapping : int64 [num_tokens] device
 * Duplicate non-negative slots in one call: which token lands is unspecified.
 * A slot >= NB*16 is skipped and sets PA_STATUS_BAD_SLOT.
 * num_tokens == 0 is a no-op.
 */
int pa_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int64_t num_tokens, const pa_shape *shape,
                         void *stream);

/*
 * pa_decode_workspace_bytes: scratch size pa_decode needs for these sizes
 * and this partition_tokens (0 = automatic), on the current device; 0 only
 * when num_seqs is 0. Negative on bad arguments.
 * With S slices (see pa_decode) and U = B * Hk units the layout is: fp32
 * partial outputs [S + U - 1][G][D], partial maxima and sums [S + U - 1][G]
 * each, then int32 (first slice, slices) records [U], each part 16-byte
 * aligned (G = H / Hk).
 */
int64_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t max_context_len, int32_t partition_tokens,
                                  const pa_shape *shape);

/*
 * pa_decode: one query token per sequence attends over its whole paged
 * context (decode-time PagedAttention; "vLLM and PagedAttention" §2
 * "Reworking the Attention Computation": K/V are loaded block by block and
 * each block's share is folded into the result).
 *
 *   out[b][h][:] = sum_p softmax_p(scale * q[b][h] . K_b[p]) V_b[p],
 *   p over 0 .. context_lens[b]-1, K_b[p] = k_cache[block_tables[b][p/16]][p%16][h/(H/Hk)]
 *
 *   out          : [B][H][D] device
 *   q            : [B][H][D] device
 *   block_tables : int32 [B][max_blocks_per_seq] device; entries past
 *                  ceil(context_lens[b]/16) are never read
 *   context_lens : int32 [B] device; 0 gives an all-zero output row
 *   max_context_len : host-side upper bound of context_lens (no device read);
 *                  it sizes the grid and the workspace. A device length above
 *                  it is clamped and sets PA_STATUS_BAD_CONTEXT.
 *   scale        : softmax scale (the sketch has none; typically 1/sqrt(D))
 *   partition_tokens : 0 = automatic. The list of (sequence, KV head,
 *                  16-token block) items is cut into S equal slices, one per
 *                  warp of a persistent grid; a (sequence, KV head) cut by
 *                  slice boundaries gets one partial (max, sum, unnormalised
 *                  O) per slice in the workspace, and a second kernel merges
 *                  them. Automatic S: the warps of all the decode CTAs the SMs
 *                  hold at once, at most one per 4 blocks of
 *                  B * Hk * ceil(max_context_len / 16). Otherwise a multiple
 *                  of 64, >= 64: S makes a slice about partition_tokens tokens
 *                  of a context of max_context_len (a smaller value means
 *                  more, smaller slices).
 *   workspace    : device scratch of >= pa_decode_workspace_bytes(...) bytes,
 *                  16-byte aligned. Its contents need no initialisation: a
 *                  call writes every partial and record before it reads it.
 *                  Calls that overlap on the GPU must not share a workspace.
 * Accumulation is fp32 whatever the dtype. bf16 output is rounded once, to
 * nearest even. Two kernel launches, the second a programmatic dependent of
 * the first.
 */
int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
              float scale, int32_t partition_tokens, void *workspace, int64_t workspace_bytes,
              const pa_shape *shape, void *stream);

/*
 * pa_decode_partials, pa_decode_merge: pa_decode's two launches, one call
 * each, with pa_decode's arguments and checks. pa_decode_partials runs the
 * partition pass: it writes the output rows of every (sequence, KV head)
 * whose blocks one warp streamed, and the partials and records of the others
 * into the workspace. pa_decode_merge, called next on the same stream with
 * the same arguments and workspace, writes the remaining rows. The pair
 * gives pa_decode's output bit for bit; other work may run on the stream
 * between them if it leaves the workspace and out alone.
 */
int pa_decode_partials(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
                       int32_t num_seqs, int32_t max_context_len, float scale, int32_t partition_tokens,
                       void *workspace, int64_t workspace_bytes, const pa_shape *shape, void *stream);
int pa_decode_merge(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                    int32_t max_context_len, float scale, int32_t partition_tokens, void *workspace,
                    int64_t workspace_bytes, const pa_shape *shape, void *stream);

/*
 * pa_prefill_chunk: causal attention for chunks of query tokens placed at a
 * context offset (chunked prefill: "vLLM — PagedAttention and Continuous
 * Batching" §5; "How vLLM Works?" §04). The chunk's K/V must already be in
 * the cache (pa_reshape_and_cache first).
 *
 * Sequence b owns query rows cu_q_lens[b] .. cu_q_lens[b+1]-1. Its chunk
 * length is q_len = cu_q_lens[b+1] - cu_q_lens[b] and its offset is
 * o = context_lens[b] - q_len. Row j of the chunk sits at absolute position
 * o + j and attends to keys 0 .. o + j (inclusive) of the paged context.
 * Chunks of any length mix in one call: a decode token is a chunk of 1, a
 * speculative verify step a chunk of a few tokens, q_len = 0 a sequence with
 * nothing to attend this step. A whole continuous-batching step is one launch.
 *
 *   out, q       : [num_q_tokens][H][D] device, num_q_tokens = cu_q_lens[B]
 *   cu_q_lens    : int32 [B + 1] device, non-decreasing, cu_q_lens[0] = 0
 *   context_lens : int32 [B] device, >= q_len
 *   max_q_len    : host-side upper bound of every q_len (checked, >= 0; the
 *                  grid is sized from num_q_tokens and num_seqs)
 *   scale        : softmax scale, > 0 (PA_ERR_INVALID_ARGUMENT otherwise)
 * q and out bf16, D = 128 only; the caches bf16, or FP8 E4M3 codes
 * (kv_fp8 = 1). Runs on the tcgen05 tensor cores with fp32 accumulation in
 * tensor memory. Probabilities enter P.V rounded to bf16; the row sums use
 * them unrounded. Over an FP8 pool the MMAs take f16 operands: each K/V tile's
 * codes are widened exactly to f16 in shared memory, q is rounded to f16 there
 * (exact for |q| in [2^-14, 65504] and for 0; outside that range q is rounded
 * or saturates to infinity), P enters P.V rounded to f16, k_scale joins the
 * softmax scale and v_scale the output. Returns PA_ERR_UNSUPPORTED for other
 * shapes.
 */
int pa_prefill_chunk(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *cu_q_lens,
                     const int32_t *context_lens, int32_t num_seqs, int32_t max_q_len, int32_t num_q_tokens,
                     float scale, const pa_shape *shape, void *stream);

/*
 * pa_copy_blocks: copy whole blocks inside the pool (copy-on-write of shared
 * prefix blocks: "vLLM — PagedAttention and Continuous Batching" §2.3,
 * "vLLM and PagedAttention" §2 "The PagedAttention Solution", "How vLLM
 * Works?" §03).
 *
 * For each pair i: block block_pairs[2i+1] of k_cache and of v_cache becomes
 * a byte copy of block block_pairs[2i]. A block is [16][Hk][D] elements.
 *   block_pairs : int64 [num_pairs][2] (src, dst), device memory
 * Destinations must be distinct and no block may be both a source and a
 * destination in one call (pairs run concurrently). An index outside
 * [0, NB) skips that pair and sets PA_STATUS_BAD_BLOCK_ID.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_pairs, int64_t num_pairs,
                   const pa_shape *shape, void *stream);

/*
 * pa_swap_blocks: move whole blocks of one pool between device memory and
 * pinned host memory, either way (preemption by swapping: "vLLM and
 * PagedAttention" §3, "How vLLM Works?" §04).
 *
 * For each pair i: block block_pairs[2i+1] of dst becomes a byte copy of block
 * block_pairs[2i] of src. Call once for K and once for V.
 *   dst, src    : device memory or pinned (page-locked) host memory; the kernel
 *                 reaches host memory through its device mapping, so the whole
 *                 swap is one launch. Pageable host memory is refused
 *                 (PA_ERR_INVALID_ARGUMENT).
 *   block_pairs : int64 [num_pairs][2] (src, dst), device or pinned host memory
 *   src_blocks, dst_blocks : blocks in each pool; block_bytes : bytes per block
 *                 (a multiple of 16)
 * Destinations must be distinct. An index outside its pool skips that pair
 * and sets PA_STATUS_BAD_BLOCK_ID.
 */
int pa_swap_blocks(void *dst, const void *src, const int64_t *block_pairs, int64_t num_pairs, int64_t src_blocks,
                   int64_t dst_blocks, int64_t block_bytes, void *stream);

/*
 * pa_decode_noalloc: pa_decode for callers that cannot allocate device memory.
 * The paper has no counterpart to this call; it is a deployment convenience.
 *
 * Some callers have no way to get a scratch buffer. Examples: code that runs
 * while a CUDA graph is being captured in a mode that forbids allocation; a
 * host engine that has reserved nearly all of HBM for its own KV pool and owns
 * every allocation; plugin code loaded into a runtime whose allocator it cannot
 * reach; a latency-critical loop where cudaMalloc's implicit synchronization is
 * not acceptable. This entry point computes exactly what pa_decode computes with
 * the same arguments. It takes no workspace: the split-context partials go to a
 * scratch array compiled into the library, PA_NOALLOC_SCRATCH_BYTES long.
 *
 *  - The array is a static device variable. Every GPU on which the library's
 *    module is loaded holds those bytes until the process exits.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current, and caches it with the
 *    device's current context. Make that first call outside any stream
 *    capture. A later call in a different context of that device (after a
 *    cudaDeviceReset, say) looks the address up again.
 *  - Requests whose partials need more than PA_NOALLOC_SCRATCH_BYTES (see
 *    pa_decode_workspace_bytes) return PA_ERR_SCRATCH_LIMIT and launch nothing.
 *    Use pa_decode with your own workspace for those, or a larger
 *    partition_tokens.
 *  - Every call on a device shares the one array, and the array keeps whatever
 *    the last call left in it. Nothing in it needs to start at zero: a call
 *    writes every partial and record before it reads it. Calls that may
 *    overlap on the GPU (different streams, or different host threads on one
 *    device) race on the array and must be serialized by the caller.
 * The library calls no cudaMalloc, cudaFree or other allocating routine here.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)

int pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
                      int32_t num_seqs, int32_t max_context_len, float scale, int32_t partition_tokens,
                      const pa_shape *shape, void *stream);

/*
 * pa_get_status: synchronize `stream`, copy the device status word of the
 * current device to *status (PA_STATUS_* flags, 0 = clean), then clear it.
 * There is one status word per device, shared by every stream and host
 * thread that uses the library on it: the flags read may have been raised by
 * a call on another stream (and a flag raised by a call still running on
 * another stream may be cleared before it is read there). Callers that need
 * per-stream attribution serialize their pa_get_status calls with the work.
 */
int pa_get_status(uint32_t *status, void *stream);

/* Static text for a pa_error code. */
const char *pa_strerror(int code);

/* cudaError_t code of the last PA_ERR_CUDA returned on this host thread (0 if none). */
int pa_last_cuda_error(void);

/* PA_ABI_VERSION of the loaded library. */
int pa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
