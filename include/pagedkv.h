/*
 * pagedkv.h - C ABI of libpagedkv.so: paged-KV decode attention for B200
 * (sm_100a) and the host block allocator that builds its block tables.
 *
 * The method ("PagedAttention: treat the cache like virtual memory",
 * "KV-Cache Management and PagedAttention"; "PagedAttention: OS Virtual Memory
 * Architecture for GPUs" and "Under the Hood: The PagedAttention CUDA Kernel",
 * "PagedAttention and KV Cache Management"): each sequence's KV cache is cut
 * into fixed-size blocks of B tokens that live anywhere in a shared pool; a
 * per-sequence block table maps logical block i (tokens iB .. iB+B-1) to its
 * physical block, and the attention kernel takes that table as an argument and
 * gathers K and V through it.
 *
 * Conventions shared by every device call
 *   - Tensors are described by pkv_tensor: a DEVICE pointer, an element type,
 *     up to 4 dims, and strides in ELEMENTS. The innermost dim must be
 *     contiguous (stride 1). The caller owns every buffer; the library never
 *     frees or keeps a pointer past the call.
 *   - Pool layout ("HND" per block): k_cache and v_cache are
 *     [num_blocks, num_kv_heads, block_size, head_dim], head_dim contiguous,
 *     strides non-decreasing outward with every byte stride a multiple of 16
 *     and the base 16-byte aligned. One (block, kv head) is one contiguous
 *     block_size * head_dim run.
 *   - Calls are asynchronous: the work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream) and
 *     nothing synchronises it. Arguments are checked on the host before any
 *     launch; a bad argument returns PKV_ERR_INVALID_ARG (or
 *     PKV_ERR_UNSUPPORTED for a valid but unimplemented shape) and launches
 *     nothing. A failed launch returns PKV_ERR_CUDA.
 *   - Device-side checks (a block id outside the pool, a context length
 *     beyond the table row, a bounded wait that ran out, a tensor-core
 *     kernel finding its shared or tensor memory placed otherwise than it
 *     assumes) never fault: the kernel records the problem in a per-device
 *     flag and carries on with safe values (or skips the work).
 *     pkv_device_error() reads and clears that flag.
 *   - Supported shapes: head_dim 64 or 128 (128 for fp8), block_size 16 or
 *     32, num_q_heads = g * num_kv_heads with 1 <= g <= 8.
 *   - Scratch: the attention calls keep their intermediate state (split-KV
 *     partials and claim words, prefix partials, multi-token partials, the
 *     longest-first sequence order) in device buffers the library owns, one
 *     set per device, grown with cudaMalloc when a call needs more. Calls
 *     that overlap on the GPU (different streams with nothing ordering
 *     them) race on those buffers: serialise them (or give each stream its
 *     own workspace through paged_attn_decode_noalloc).
 *
 * The host allocator calls touch no device memory and are not thread-safe
 * per handle (one handle per scheduler thread).
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_F16 = 0,       /* IEEE binary16 */
  PKV_BF16 = 1,      /* bfloat16 */
  PKV_FP8_E4M3 = 2,  /* OCP fp8 E4M3 codes, stored as bytes */
  PKV_I32 = 3,
  PKV_I64 = 4,
  PKV_F32 = 5
} pkv_dtype;

typedef struct {
  void* data;        /* device pointer */
  int32_t dtype;     /* pkv_dtype */
  int32_t ndim;      /* 1..4 */
  int64_t shape[4];
  int64_t stride[4]; /* elements */
} pkv_tensor;

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = -1,
  PKV_ERR_UNSUPPORTED = -2,
  PKV_ERR_OOM = -3,          /* allocator: not enough free blocks */
  PKV_ERR_UNKNOWN_SEQ = -4,  /* allocator: no such sequence */
  PKV_ERR_EXISTS = -5,       /* allocator: sequence id already in use */
  PKV_ERR_DOUBLE_FREE = -6,  /* allocator: reference count would drop below 0 */
  PKV_ERR_CUDA = -7,         /* a CUDA runtime call failed */
  PKV_ERR_DEVICE_CHECK = -8, /* a kernel recorded a bad index or a wait that ran out */
  PKV_ERR_WORKSPACE = -9,    /* caller-provided workspace too small */
  PKV_ERR_SCRATCH_LIMIT = -10 /* needs more than the library's static scratch */
} pkv_status;

/* Text for a status code (static storage, never NULL). */
const char* pkv_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int pkv_version(void);

/* ------------------------------------------------------------------------ */
/* Decode attention                                                         */
/* ------------------------------------------------------------------------ */

/*
 * paged_attn_decode - one decode step of attention over a paged KV cache.
 *
 * Defined by "Under the Hood: The PagedAttention CUDA Kernel" ("PagedAttention
 * and KV Cache Management") and the block-table diagram of "PagedAttention:
 * treat the cache like virtual memory" ("KV-Cache Management and
 * PagedAttention"). For every sequence s and query head i, with kv head
 * h = i / g and L = context_lens[s]:
 *     K_s[t] = k_cache[block_tables[s][t / B], h, t % B, :]   (same for V)
 *     out[s, i, :] = softmax_t(scale * <q[s, i, :], K_s[t]>) . V_s
 * over t = 0 .. L-1. L = 0 gives out = 0. Slots past L in the last block and
 * table entries past ceil(L/B) are never read into the result (they may hold
 * anything, NaN included).
 *
 *   q            [S, Hq, D] f16 | bf16, read only
 *   k_cache      [NB, Hk, B, D], same dtype as q
 *   v_cache      [NB, Hk, B, D], same dtype as q
 *   block_tables [S, MB] int32 physical block ids; entries >= ceil(L/B) ignored
 *   context_lens [S] int32, 0 <= L <= MB * B (the new token included)
 *   num_kv_heads Hk (must equal k_cache.shape[1])
 *   scale        softmax scale (usually 1/sqrt(D))
 *   block_size   B (must equal k_cache.shape[2])
 *   out          [S, Hq, D], same dtype as q, written
 *
 * Uses a per-device workspace owned by the library: the first call on a
 * device (or one needing more) allocates it with cudaMalloc and zeroes it
 * on `stream`; a larger one replaces the old buffer, which is released with
 * cudaFree (that waits for all work on the device, so no stream still uses
 * it). Either makes that call synchronise the device and keeps it out of
 * stream capture: make a first call of the largest shape before capturing.
 * Later calls reuse the buffer and do not synchronise. Calls that share a
 * device and overlap on the GPU must use paged_attn_decode_ex with separate
 * workspaces.
 */
int paged_attn_decode(const pkv_tensor* q, const pkv_tensor* k_cache, const pkv_tensor* v_cache,
                      const pkv_tensor* block_tables, const pkv_tensor* context_lens,
                      int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                      void* stream);

/*
 * paged_attn_decode_fp8 - as paged_attn_decode with an fp8-e4m3 cache.
 * An fp8 cache halves the bytes per element ("Planning capacity when context
 * gets long", "KV-Cache Management and PagedAttention"; "The KV Cache Size
 * Equation", "PagedAttention and KV Cache Management").
 *
 *   k_cache, v_cache  [NB, Hk, B, D] PKV_FP8_E4M3 codes
 *   k_scale, v_scale  [Hk] f32 device: element value = decode(code) * scale[h]
 *   q, out            f16 | bf16 (q is rounded to f16 for the dot products;
 *                     a bf16 row of one head whose largest magnitude is 2^16
 *                     or more is first scaled by a power of two, which its
 *                     logit scale takes back, so it does not overflow)
 */
int paged_attn_decode_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                          const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                          const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                          const pkv_tensor* context_lens, int num_kv_heads, float scale,
                          int block_size, pkv_tensor* out, void* stream);

/*
 * Bytes of workspace a decode with these sizes needs on `device`
 * (split-KV partial results, one small header). Depends on the device's SM
 * count, not on the context lengths.
 */
size_t paged_attn_decode_workspace_bytes(int num_q_heads, int num_kv_heads, int head_dim,
                                         int block_size, int cache_dtype, int device);

/*
 * paged_attn_decode_ex - the general form: k_scale / v_scale are NULL for a
 * 16-bit cache and required for fp8; `workspace` is a caller-owned device
 * buffer of at least paged_attn_decode_workspace_bytes() bytes (16-byte
 * aligned), else PKV_ERR_WORKSPACE. Zero-fill it once before its first use
 * (e.g. cudaMemset): it holds the split-KV work-claiming state, which every
 * call leaves zeroed again. The workspace must not be used by another call
 * until this one has finished on the GPU; after a PKV_ERR_DEVICE_CHECK from
 * a call that used it, zero it again. With an fp8 cache, and a batch with at
 * least as many (sequence, kv head) units as the call has warp ranges, the
 * workspace also carries from call to call how the work was split: each
 * call learns from its warps' times where the next call should cut the
 * work (results do not depend on it; a workspace shared by very different
 * batches only balances less well).
 *
 * flags: 0, or PKV_DECODE_DETERMINISTIC. By default a warp that runs out of
 * work takes over part of another warp's remaining blocks, so where a
 * sequence's context is cut between warps (and so the order in which its
 * partial sums are added) changes from call to call with the timing: results
 * agree to rounding, not bit for bit. PKV_DECODE_DETERMINISTIC cuts the
 * work only where the static split puts the cuts and merges the pieces in a
 * fixed order, so identical calls on the same device give identical bits
 * (the slowest SMs then set the time: usually a little slower). Other bits:
 * PKV_ERR_INVALID_ARG.
 */
#define PKV_DECODE_DETERMINISTIC 1u
int paged_attn_decode_ex(const pkv_tensor* q, const pkv_tensor* k_cache,
                         const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                         const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                         const pkv_tensor* context_lens, int num_kv_heads, float scale,
                         int block_size, pkv_tensor* out, void* workspace,
                         size_t workspace_bytes, unsigned flags, void* stream);

/*
 * paged_attn_prefill - causal attention of several new tokens per sequence
 * over the paged cache: a prompt, or a chunk of one, whose K/V were written
 * to the blocks allocated for it ("How Block Paging Operates During
 * Generation": a request's prompt gets its blocks when it starts; "Dynamic
 * Request Insertion": a waiting request's prefill joins the running
 * iteration), or speculative tokens being verified. Sequence s has
 * n_s = q_start[s + 1] - q_start[s] new tokens, the last n_s of its
 * L_s = context_lens[s] (0 <= n_s <= L_s); query row q_start[s] + j is the
 * token at position L_s - n_s + j and attends to positions 0 .. L_s - n_s + j.
 * n_s = 1 for every s is the decode step.
 *
 *   q             device [T, Hq, D] f16 | bf16, rows grouped by sequence
 *   k_cache, v_cache, block_tables, context_lens, num_kv_heads, scale,
 *   block_size    as paged_attn_decode (16-bit caches; fp8 caches:
 *                 paged_attn_prefill_fp8)
 *   q_start       device int32 [S + 1], non-decreasing, q_start[S] <= T
 *   max_q_tokens  host int >= every n_s (sizes the launch)
 *   out           device [T, Hq, D] like q; rows of tokens in no sequence
 *                 are left untouched
 * Kernels, by query rows per (sequence, kv head) (new tokens x group heads):
 * up to 64, one CTA per (sequence, kv head, 16 / 32 / 64 query columns) with
 * warp MMAs, a column being one query head of one new token (the chunk's
 * columns share every K/V tile read); from 64 (D = 128, scale > 0), 128-row
 * tiles on the tensor cores, one or two per CTA, sequences taken longest
 * context first (a one-CTA ordering pass runs before them when S <= 1024
 * and the grid is more than one wave).
 * With max_q_tokens = 1 and T = S (one new token per sequence) the call is
 * the decode step and runs the decode kernels; q_start, which can then only
 * be 0, 1, ..., S, is not read. Asynchronous on `stream`; an inconsistent
 * q_start / context_lens row or block id is flagged (PKV_ERR_DEVICE_CHECK)
 * and that row skipped.
 */
int paged_attn_prefill(const pkv_tensor* q, const pkv_tensor* k_cache, const pkv_tensor* v_cache,
                       const pkv_tensor* block_tables, const pkv_tensor* context_lens,
                       const pkv_tensor* q_start, int max_q_tokens, int num_kv_heads, float scale,
                       int block_size, pkv_tensor* out, void* stream);

/*
 * paged_attn_prefill_fp8 - paged_attn_prefill over an fp8-e4m3 cache:
 * k_cache / v_cache PKV_FP8_E4M3 codes [NB, Hk, B, 128], k_scale / v_scale
 * f32 device [Hk] (element value = decode(code) * scale[h]); q / out f16 |
 * bf16, q rounded to f16 for the dot products as in paged_attn_decode_fp8
 * (a bf16 row of one head reaching 2^16 first scaled by a power of two that
 * its logit scale takes back). Every row count runs on the warp-MMA kernel
 * (codes widened to f16 in registers; a tcgen05 f16 product takes both
 * operands in one 16-bit type); one new token per sequence is the fp8
 * decode step. head_dim 128, block_size 16 or 32, else PKV_ERR_UNSUPPORTED;
 * other arguments and errors as paged_attn_prefill.
 */
int paged_attn_prefill_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                           const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                           const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                           const pkv_tensor* context_lens, const pkv_tensor* q_start,
                           int max_q_tokens, int num_kv_heads, float scale, int block_size,
                           pkv_tensor* out, void* stream);

/*
 * swap_out_blocks / swap_in_blocks - the device half of preemption by
 * swapping ("Preemption and eviction", KV-Cache Management and
 * PagedAttention; "Preemption & GPU Swapping", PagedAttention and KV Cache
 * Management): blocks of both pools to page-locked host memory and back,
 * bit-exact, so a preempted sequence can resume in other blocks
 * (pkv_seq_swap_out / pkv_seq_swap_in pick them).
 *
 *   k_cache, v_cache  device [NB, Hk, B, D] pools, same type (f16, bf16 or fp8
 *                     codes; bytes are copied), same strides, rows 16-byte
 *                     multiples
 *   blocks            device int32 [n]: block ids, in record order
 *   host_dst/host_src page-locked host memory mapped into the device's
 *                     address space (cudaHostAlloc, or torch pin_memory),
 *                     16-byte aligned, host_bytes >= n * record bytes;
 *                     record i = block blocks[i]'s K tile [Hk, B, D]
 *                     (row-major) then its V tile, 2 * Hk * B * D * e bytes
 * The kernel reads or writes the host memory itself through its device
 * mapping (no staging copy). Asynchronous on `stream`; the host buffer must
 * stay allocated until the stream reaches that point. PKV_ERR_INVALID_ARG
 * for pageable or unmapped host memory or a short buffer; a block id outside
 * the pool is flagged (PKV_ERR_DEVICE_CHECK) and its record skipped.
 */
int swap_out_blocks(const pkv_tensor* k_cache, const pkv_tensor* v_cache, const pkv_tensor* blocks,
                    void* host_dst, size_t host_bytes, void* stream);
int swap_in_blocks(const void* host_src, size_t host_bytes, const pkv_tensor* blocks,
                   pkv_tensor* k_cache, pkv_tensor* v_cache, void* stream);

/*
 * paged_attn_decode_cascade - paged_attn_decode for a batch whose sequences
 * share prompt prefixes, reading each shared prefix block once per group
 * instead of once per sequence. Prefix sharing: "PagedAttention: treat the
 * cache like virtual memory" (KV-Cache Management and PagedAttention) and
 * "Shared System Prompts & Prefix Caching" (PagedAttention and KV Cache
 * Management); the result is the attention paged_attn_decode defines (the
 * softmax over a sequence's tokens is split into its prefix and the rest and
 * recombined with the log-sum-exp rule), equal to it up to rounding order.
 *
 * Same q, caches (16-bit), block_tables, context_lens, num_kv_heads,
 * scale, block_size, out and stream as paged_attn_decode, plus a grouping of
 * the batch (pkv_prefix_groups computes one from the tables on the host):
 *   prefix_blocks  device int32 [S]: the leading table entries sequence s
 *                  shares with its group (whole, full blocks), 0 if s is in
 *                  no group
 *   group_start    device int32 [num_groups + 1], group_members device
 *                  int32 [M]: group g's members (batch rows) are
 *                  group_members[group_start[g] .. group_start[g + 1])
 *   num_groups, max_group_size (members of the largest group),
 *   max_prefix_blocks (largest prefix_blocks): host ints sizing the launch
 * Contract: a member's first prefix_blocks entries equal those of its
 * group's first member, are full (prefix_blocks * block_size <= length), and
 * are not written by this step; prefix_blocks[s] > 0 exactly for members.
 * Rows breaking it are flagged (PKV_ERR_DEVICE_CHECK) where the kernels can
 * see it, else their output rows are undefined.
 *
 * Kernels, in stream order: decode over each sequence's tokens after its
 * prefix (sequences with a prefix leave fp32 partials), the split-KV merge,
 * one prefix pass per (group, kv head, 64 query columns, prefix-block chunk)
 * in which every query head of every member attends the shared blocks, and a
 * final merge writing out. Uses a library-owned device buffer (grown with
 * cudaMalloc when a larger batch needs it; fp32 partials of S * Hq rows plus
 * the prefix chunks). fp8 caches: paged_attn_decode_cascade_fp8.
 */
int paged_attn_decode_cascade(const pkv_tensor* q, const pkv_tensor* k_cache,
                              const pkv_tensor* v_cache, const pkv_tensor* block_tables,
                              const pkv_tensor* context_lens, const pkv_tensor* prefix_blocks,
                              const pkv_tensor* group_start, const pkv_tensor* group_members,
                              int num_groups, int max_group_size, int max_prefix_blocks,
                              int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                              void* stream);

/*
 * paged_attn_decode_cascade_fp8 - paged_attn_decode_cascade over an
 * fp8-e4m3 cache: k_cache / v_cache PKV_FP8_E4M3 codes [NB, Hk, B, 128],
 * k_scale / v_scale f32 device [Hk] (element value = decode(code) *
 * scale[h]), q / out f16 | bf16 with the rounding of paged_attn_decode_fp8
 * (q to f16 for the dot products, a bf16 row of one head reaching 2^16
 * first scaled by a power of two that its logit scale takes back). The
 * shared prefix is still read once per group; the prefix pass widens the
 * codes in registers as the decode does. head_dim 128, block_size 16 or 32,
 * else PKV_ERR_UNSUPPORTED; other arguments and errors as
 * paged_attn_decode_cascade.
 */
int paged_attn_decode_cascade_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                                  const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                                  const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                                  const pkv_tensor* context_lens, const pkv_tensor* prefix_blocks,
                                  const pkv_tensor* group_start, const pkv_tensor* group_members,
                                  int num_groups, int max_group_size, int max_prefix_blocks,
                                  int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                                  void* stream);

/*
 * paged_attn_decode_noalloc - paged_attn_decode / paged_attn_decode_fp8 for
 * callers that cannot allocate device memory when they call: for example an
 * engine that hands almost all of HBM to its own KV-block pool at start-up
 * (a late cudaMalloc would fail or fragment that pool), or a caller whose
 * latency budget cannot absorb the device synchronisation cudaMalloc
 * implies. The pages have no counterpart of this call; it is a property of
 * this library, not of the method.
 *
 * Same arguments and results as paged_attn_decode_ex without the workspace:
 * k_scale / v_scale are NULL for a 16-bit cache and required for fp8. The
 * split-KV scratch lives in a static device array of
 * PKV_NOALLOC_SCRATCH_BYTES bytes that every GPU loading this library keeps
 * until the process exits. The call allocates nothing: it calls no
 * cudaMalloc / cudaFree and no allocating library routine.
 *
 *   - The first call on each device looks up that array's device address
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture on the device.
 *   - A shape whose minimum scratch would exceed the limit (it grows with
 *     the device's SM count, the query-head group g and head_dim, not with
 *     the context lengths) returns PKV_ERR_SCRATCH_LIMIT and launches
 *     nothing.
 *   - All calls on a device share the one array and it keeps the last
 *     call's contents; each call first zeroes the part that must start at
 *     zero (the work-claiming state, a few KB, with cudaMemsetAsync on
 *     `stream`). Calls that overlap on the GPU (different streams, no
 *     ordering between them) race on the array and give wrong results:
 *     serialise them.
 *   - When the default split-KV scratch does not fit, the call keeps fewer
 *     slots for rebalancing work between warps (same results, possibly a
 *     little slower).
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)
int paged_attn_decode_noalloc(const pkv_tensor* q, const pkv_tensor* k_cache,
                              const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                              const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                              const pkv_tensor* context_lens, int num_kv_heads, float scale,
                              int block_size, pkv_tensor* out, void* stream);

/* ------------------------------------------------------------------------ */
/* Cache writes and block copies                                            */
/* ------------------------------------------------------------------------ */

/*
 * reshape_and_cache - store each new token's K and V rows in its slot.
 * During generation a token is written into its sequence's current block
 * ("How Block Paging Operates During Generation", "PagedAttention and KV
 * Cache Management"). Slot = physical_block * B + offset:
 *     k_cache[slot / B, h, slot % B, :] = k[t, h, :]   (same for v)
 * for every t with slot_mapping[t] >= 0 (negative = padding, skipped).
 *
 *   k, v          [T, Hk, D] same dtype as the caches (f16 | bf16)
 *   k_cache, v_cache [NB, Hk, B, D], written
 *   slot_mapping  [T] int64; slots must be distinct and < NB * B
 * Bit-exact copy. A slot >= NB * B is skipped and flagged as a device check.
 */
int reshape_and_cache(const pkv_tensor* k, const pkv_tensor* v, pkv_tensor* k_cache,
                      pkv_tensor* v_cache, const pkv_tensor* slot_mapping, void* stream);

/*
 * reshape_and_cache_fp8 - as reshape_and_cache into an fp8-e4m3 pool: stores
 * the e4m3 code of the fp32 quotient x / scale[h], rounded to nearest even
 * and saturated to +-448 (NaN stays NaN).
 *
 *   k, v          [T, Hk, D] f16 | bf16
 *   k_cache, v_cache [NB, Hk, B, D] PKV_FP8_E4M3
 *   k_scale, v_scale [Hk] f32 device
 */
int reshape_and_cache_fp8(const pkv_tensor* k, const pkv_tensor* v, pkv_tensor* k_cache,
                          pkv_tensor* v_cache, const pkv_tensor* slot_mapping,
                          const pkv_tensor* k_scale, const pkv_tensor* v_scale, void* stream);

/*
 * copy_blocks - device half of copy-on-write ("Parallel Sampling & Beam Search
 * via Copy-on-Write", "PagedAttention and KV Cache Management"): for each
 * (src, dst) row of `pairs`, block dst of both caches becomes a bit-exact copy
 * of block src (all heads, all B slots).
 *
 *   k_cache, v_cache [NB, Hk, B, D] any element type (same for both)
 *   pairs         [n, 2] int32 device; every dst distinct and no dst also a
 *                 src in the same call (the allocator's copy-on-write pairs
 *                 satisfy this), so that every copy reads the pool as it was
 *                 before the call whatever order they run in. A pair whose
 *                 dst is another pair's src or dst, or whose src is another
 *                 pair's dst, is not copied and is flagged
 *                 (PKV_ERR_DEVICE_CHECK); the other pairs are copied. Ids
 *                 outside the pool are skipped and flagged.
 */
int copy_blocks(pkv_tensor* k_cache, pkv_tensor* v_cache, const pkv_tensor* pairs,
                void* stream);

/*
 * pkv_device_error - synchronises `device` and returns PKV_ERR_DEVICE_CHECK
 * if any kernel of this library flagged a device-side check since the last
 * call (then clears the flag), else PKV_OK. Returns PKV_ERR_CUDA if the
 * synchronisation itself fails.
 */
int pkv_device_error(int device);

/* ------------------------------------------------------------------------ */
/* Host block allocator                                                     */
/* ------------------------------------------------------------------------ */
/*
 * Semantics of "Hands-On Implementation: Building a PagedAttention Block
 * Allocator in Python" ("PagedAttention and KV Cache Management"): a pool of
 * num_blocks blocks of block_size slots; new blocks come from the HEAD of the
 * free list and released blocks go to its TAIL; a sequence of n tokens holds
 * ceil(n / B) blocks; forking shares every block (reference count + 1);
 * freeing drops one reference per block; a block is copied on write when a
 * sequence must write into a block another sequence still references. Each
 * call either succeeds or returns an error and changes nothing.
 *
 * Sequence ids are caller-chosen int64 values.
 */

/* Create a pool. initial_free_order: NULL for 0..num_blocks-1, else a
 * permutation of the block ids giving the initial free-list order (host). */
int pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                     void** handle);
void pkv_alloc_destroy(void* handle);

/* New sequence holding num_tokens tokens in ceil(num_tokens / B) fresh
 * blocks. PKV_ERR_EXISTS, PKV_ERR_OOM. */
int pkv_seq_allocate(void* handle, int64_t seq, int32_t num_tokens);

/* Reserve the slot of the sequence's next token. *slot gets the flat slot
 * (block * B + offset). If the token must go into a block shared with
 * another sequence, a fresh block replaces it in this sequence's table and
 * *cow_src / *cow_dst name the block copy the device must do first (see
 * copy_blocks); otherwise both are -1. A full last block (shared or not)
 * gets a new block after it. PKV_ERR_UNKNOWN_SEQ, PKV_ERR_OOM. */
int pkv_seq_append_slot(void* handle, int64_t seq, int64_t* slot, int32_t* cow_src,
                        int32_t* cow_dst);

/* dst shares every block of src (zero-copy fork). PKV_ERR_UNKNOWN_SEQ,
 * PKV_ERR_EXISTS. */
int pkv_seq_fork(void* handle, int64_t src, int64_t dst);

/* Drop the sequence and one reference on each of its blocks, in table order;
 * a block reaching 0 returns to the tail of the free list. Unknown seq:
 * PKV_OK, nothing done. */
int pkv_seq_free(void* handle, int64_t seq);

/* Tokens held by seq (>= 0), or PKV_ERR_UNKNOWN_SEQ. */
int64_t pkv_seq_num_tokens(void* handle, int64_t seq);

/* Copy seq's block table into table[0 .. cap) (host); returns the number of
 * blocks (which may exceed cap: only cap entries are written), or an error. */
int pkv_seq_block_table(void* handle, int64_t seq, int32_t* table, int32_t cap);

/* Build the decode inputs for n sequences, on the host: row i of `table`
 * (n x max_blocks, row-major) gets seqs[i]'s block ids padded with -1, and
 * lens[i] its token count. PKV_ERR_UNKNOWN_SEQ; PKV_ERR_INVALID_ARG if a
 * table does not fit in max_blocks. */
int pkv_build_block_tables(void* handle, const int64_t* seqs, int32_t n, int32_t* table,
                           int32_t max_blocks, int32_t* lens);

/* Pool statistics: free blocks, used blocks (refcount > 0), shared blocks
 * (refcount > 1), tokens stored (each physical slot counted once). Any
 * output pointer may be NULL. */
int pkv_alloc_stats(void* handle, int32_t* free_blocks, int32_t* used_blocks,
                    int32_t* shared_blocks, int64_t* tokens);

/* Reference count of one block (>= 0) or PKV_ERR_INVALID_ARG. */
int pkv_block_refcount(void* handle, int32_t block);

/* Preemption by swapping ("Preemption and eviction", KV-Cache Management and
 * PagedAttention; "Preemption & GPU Swapping", PagedAttention and KV Cache
 * Management).
 *
 * pkv_seq_swap_out: writes the sequence's blocks, in table order, to
 * blocks[0 .. *n) (cap entries available) and drops this sequence's reference
 * on each (a block whose count reaches 0 returns to the tail of the free
 * list). Copy those blocks to host memory (swap_out_blocks) before anything
 * reuses them. The sequence keeps its token count and becomes swapped out:
 * every call but pkv_seq_free (which forgets it) and pkv_seq_swap_in answers
 * PKV_ERR_UNKNOWN_SEQ for it, and its id stays taken (PKV_ERR_EXISTS).
 * pkv_seq_swap_in: takes ceil(tokens / block_size) fresh blocks for a
 * swapped-out sequence, writes them to blocks[0 .. *n) in table order (fill
 * them with swap_in_blocks) and makes the sequence live again.
 * Errors change nothing: PKV_ERR_UNKNOWN_SEQ, PKV_ERR_INVALID_ARG (cap too
 * small, null pointer), PKV_ERR_OOM (not enough free blocks). */
int pkv_seq_swap_out(void* handle, int64_t seq, int32_t* blocks, int32_t cap, int32_t* n);
int pkv_seq_swap_in(void* handle, int64_t seq, int32_t* blocks, int32_t cap, int32_t* n);

/* Utilisation figures of the pool ("Managing the KV cache": blocks stored with
 * sharing versus storing each request's blocks separately, and the memory
 * that saves; tokens held over the slots of used blocks): *table_blocks =
 * the sum of all live sequences' table lengths (the blocks a pool without
 * sharing would hold), *sequences = live sequences. With pkv_alloc_stats'
 * used blocks U and tokens T: saved = 1 - U / table_blocks, utilisation =
 * T / (U * block_size), and U * block_size - T <= (block_size - 1) *
 * sequences (at most one partly filled block per sequence). */
int pkv_alloc_utilisation(void* handle, int64_t* table_blocks, int32_t* sequences);

/* A new sequence whose first num_blocks table entries are the given blocks
 * (blocks in use, e.g. a prefix-cache match: one more reference each) and
 * whose remaining ceil(num_tokens / block_size) - num_blocks blocks are
 * fresh; num_blocks * block_size <= num_tokens. PKV_ERR_EXISTS,
 * PKV_ERR_INVALID_ARG, PKV_ERR_OOM change nothing. */
int pkv_seq_allocate_prefix(void* handle, int64_t seq, const int32_t* blocks, int32_t num_blocks,
                            int32_t num_tokens);

/* Prefix cache over an allocator ("RadixAttention — reuse a shared prefix";
 * "Shared System Prompts & Prefix Caching"): a radix tree whose nodes are
 * full blocks, keyed by their block_size token ids; the cache holds one
 * reference on each node's block, so cached blocks outlive the sequences
 * that wrote them. pkv_cache_destroy drops those references; destroying the
 * allocator first detaches its caches (their calls then return
 * PKV_ERR_INVALID_ARG; destroy them still). Host-only; not thread-safe (one
 * caller at a time, allocator and caches together).
 *   pkv_cache_insert: walk sequence seq's first n / block_size full blocks
 *     (tokens: its first n token ids); a block whose tokens are already
 *     cached on that path is left alone, others become nodes. *added = nodes
 *     added. PKV_ERR_UNKNOWN_SEQ, PKV_ERR_INVALID_ARG (n above the sequence's
 *     token count); PKV_ERR_OOM may leave a leading part cached.
 *   pkv_cache_match: the blocks of the longest run of leading full blocks of
 *     tokens[0..n) found in the tree (at most cap) into blocks, *matched =
 *     their count; every node on the run counts as used now.
 *   pkv_cache_evict: up to n times, release the least recently used leaf
 *     whose block only the cache references (ties: the older node), its
 *     block returning to the free list; *num_freed blocks written to freed.
 *   The use clock advances once per insert and per match.
 *   pkv_cache_nodes: cached blocks (>= 0). */
int pkv_cache_create(void* alloc, void** cache);
void pkv_cache_destroy(void* cache);
int pkv_cache_insert(void* cache, int64_t seq, const int32_t* tokens, int32_t n, int32_t* added);
int pkv_cache_match(void* cache, const int32_t* tokens, int32_t n, int32_t* blocks, int32_t cap,
                    int32_t* matched);
int pkv_cache_evict(void* cache, int32_t n, int32_t* freed, int32_t* num_freed);
int pkv_cache_nodes(void* cache);

/* Shared-prefix groups of a decode batch, for paged_attn_decode_cascade.
 * Prefix sharing: "PagedAttention: treat the cache like virtual memory"
 * (KV-Cache Management and PagedAttention) and "Shared System Prompts & Prefix
 * Caching" (PagedAttention and KV Cache Management): requests that start with
 * the same prompt point their block tables at the same physical blocks.
 *
 * Rows (batch positions) whose first block is full (lens[r] >= block_size)
 * are bucketed by that first block id, buckets in order of their lowest row,
 * rows ascending. A bucket of at least min_members rows is a group; its
 * prefix is the longest run of leading table columns j that hold the same
 * block in every member and are full in every member ((j + 1) * block_size
 * <= lens[r]).
 *   tables         host int32 [S, width], row-major (row stride width)
 *   lens           host int32 [S]
 *   group_start    host int32 [S + 1] out: group g's members are
 *                  members[group_start[g] .. group_start[g + 1])
 *   members        host int32 [S] out: rows, grouped
 *   prefix_blocks  host int32 [S] out: the shared prefix of the row's group in
 *                  blocks, 0 for rows in no group
 *   num_groups, num_members  out: G and M
 * Pure host function, no state. PKV_ERR_INVALID_ARG on a null pointer,
 * S < 0, width < 1, block_size < 1 or min_members < 1; PKV_ERR_OOM if host
 * memory runs out. */
int pkv_prefix_groups(const int32_t* tables, int32_t S, int32_t width, const int32_t* lens,
                      int32_t block_size, int32_t min_members, int32_t* group_start,
                      int32_t* members, int32_t* prefix_blocks, int32_t* num_groups,
                      int32_t* num_members);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
