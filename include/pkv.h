/*
 * pkv.h -- C ABI of libpkv, the B200 (sm_100a) paged KV-cache decode path.
 *
 * The operations follow the PagedAttention description in "Memory Optimization in LLM
 * Serving with PagedAttention" (sections "How PagedAttention Works" and "Advanced
 * Capabilities: Memory Sharing with Copy-on-Write") and "vLLM and PagedAttention: How Ideas
 * from Operating Systems Accelerated LLM Inference": the KV cache is a pool of fixed-size
 * physical blocks of 16 (or 32) tokens, each sequence reaches its tokens through a block
 * table, a custom kernel gathers the scattered blocks to compute attention, and shared blocks
 * are copied before a sequence writes into them.
 *
 * Conventions (every function):
 *   - Returns pkv_status; PKV_OK is 0.  On failure pkv_last_error() (per calling thread)
 *     describes the first problem found.  Nothing is launched when host-side validation fails.
 *   - Tensor pointers are DEVICE pointers owned by the caller unless a parameter says "host".
 *     The library allocates no device memory on these paths; scratch space is passed in.
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default stream).  Launches
 *     are asynchronous; the calls return once the kernels are queued.
 *   - dtype is one of pkv_dtype; q, out, the pools and the new K/V all use the same dtype.
 *   - Pool layout: k_pool and v_pool are row-major [num_blocks][num_kv_heads][block_size]
 *     [head_dim], so one (block, kv head) is a contiguous block_size*head_dim run.  With
 *     B = block_size (16 or 32), token t of sequence s is at block
 *     block_tables[s*max_blocks_per_seq + t/B], offset t%B.  A slot number names (block,
 *     offset) as block*B + offset.
 *   - Device-side checks: values only the GPU sees (context lengths, table entries, slots,
 *     block ids) are range-checked by the kernels before any access.  A bad value is skipped
 *     (never dereferenced) and sets a bit in the device fault word that
 *     pkv_device_faults() reads.  Outputs that depended on a bad value are unspecified.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID = 1,      /* bad argument (null pointer, shape, alignment, range)   */
    PKV_ERR_OOM = 2,          /* block manager: not enough free blocks; state unchanged */
    PKV_ERR_UNSUPPORTED = 3,  /* valid but not built: head_dim, dtype, block size       */
    PKV_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed                   */
    PKV_ERR_NOT_FOUND = 5     /* block manager: unknown sequence id                     */
} pkv_status;

/* PKV_FP8_E4M3 names FP8 pools in kv_copy_blocks / kv_swap_* (1-byte elements); the FP8
 * decode and write take the q / new-value dtype in desc->dtype instead. */
typedef enum pkv_dtype { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2, PKV_FP8_E4M3 = 3 } pkv_dtype;

/* Bits of the device fault word. */
#define PKV_FAULT_BAD_LEN   0x1u  /* context_lens[s] outside [1, max_blocks_per_seq*16]  */
#define PKV_FAULT_BAD_BLOCK 0x2u  /* block table entry outside [0, num_blocks)          */
#define PKV_FAULT_BAD_SLOT  0x4u  /* slot outside [0, num_blocks*16) and not -1; in the  */
                                  /* fused write-and-decode calls, a slot that is not    */
                                  /* -1 and not the one of position context_lens[s]-1    */
#define PKV_FAULT_BAD_PAIR  0x8u  /* copy pair naming a block outside [0, num_blocks)   */
#define PKV_FAULT_TIMEOUT   0x10u /* a bounded wait on a shared-memory barrier gave up  */
#define PKV_FAULT_DUPLICATE 0x20u /* kv_write(_fp8): a slot named by two tokens of the   */
                                  /* call; kv_copy_blocks: a destination named by two    */
                                  /* pairs, or one that is also a source; kv_swap_*: a   */
                                  /* destination named by two pairs.  Those entries are  */
                                  /* skipped, the others carried out                      */
#define PKV_FAULT_BAD_SCALE 0x40u /* FP8: a K or V scale that is not finite and > 0     */

/* Shape of one decode batch and of the pools it reads. */
typedef struct pkv_attn_desc {
    int32_t num_seqs;            /* S                                                   */
    int32_t num_q_heads;         /* H_q                                                 */
    int32_t num_kv_heads;        /* H_kv; H_q % H_kv == 0, query head h reads kv head   */
                                 /* h / (H_q / H_kv)                                    */
    int32_t head_dim;            /* D: 64 or 128                                        */
    int32_t block_size;          /* tokens per block B: 16 or 32                        */
    int32_t num_blocks;          /* NB, physical blocks in each pool                    */
    int32_t max_blocks_per_seq;  /* row stride of block_tables                          */
    int32_t dtype;               /* pkv_dtype                                           */
    int32_t partition_tokens;    /* context split for long sequences: 0 = library's     */
                                 /* choice, else a multiple of 16                       */
} pkv_attn_desc;

/* Last error message of the calling thread ("" if none).  Never NULL. */
const char *pkv_last_error(void);

/* Library version string. */
const char *pkv_version(void);

/*
 * Scratch bytes paged_attn_decode needs for split-context partial results (0 when no
 * sequence of this shape can span more than one partition).  Depends only on the
 * descriptor.  Returns 0 and sets the last error on an invalid descriptor.
 */
size_t pkv_attn_workspace_bytes(const pkv_attn_desc *desc);

/*
 * Single-token decode attention over the paged KV cache ("Memory Optimization in LLM Serving
 * with PagedAttention", section "How PagedAttention Works": the kernel gathers the scattered
 * KV blocks through the block table to compute attention).  For every sequence s and query
 * head h, with L = context_lens[s] and kv head hk = h / (H_q / H_kv):
 *     x_t = scale * <q[s,h,:], K_t>   for t in [0, L), K_t read through the block table
 *     out[s,h,:] = sum_t softmax(x)_t * V_t
 * accumulated in fp32 and rounded once to dtype.
 *   q            [S, H_q, D] dtype
 *   k_pool/v_pool [NB, H_kv, B, D] dtype, 16-byte aligned
 *   block_tables [S, max_blocks_per_seq] int32; only the first ceil(L/16) entries of a row
 *                are read
 *   context_lens [S] int32, each in [1, max_blocks_per_seq*B] (checked on the device)
 *   out          [S, H_q, D] dtype
 *   workspace    at least pkv_attn_workspace_bytes(desc) bytes, 256-byte aligned (may be
 *                NULL when that is 0); overwritten; calls that share it must not overlap
 * Sequences longer than the partition size are split; each partition is computed
 * independently and a second kernel merges the partitions by log-sum-exp.
 */
pkv_status paged_attn_decode(const pkv_attn_desc *desc, const void *q, const void *k_pool,
                             const void *v_pool, const int32_t *block_tables,
                             const int32_t *context_lens, float scale, void *out,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Scatter each new token's K and V into its slot ("Memory Optimization in LLM Serving with
 * PagedAttention", section "How PagedAttention Works": blocks are filled on demand as
 * generation proceeds).  For token t and kv head h:
 *     k_pool[slot/16, h, slot%16, :] = k_new[t, h, :]   (and the same for V)
 * bytes copied unchanged.  slot_mapping[t] == -1 skips token t.
 *   k_new/v_new  [num_tokens, H_kv, D] dtype
 *   slot_mapping [num_tokens] int64, distinct values in [0, NB*B) or -1
 * Checked on the device: a slot outside the pool is skipped (PKV_FAULT_BAD_SLOT); a slot
 * that two or more tokens of the call name is skipped for all of them
 * (PKV_FAULT_DUPLICATE), so the pools never depend on which write lands last.  The check
 * compares every slot with every other, num_tokens^2 comparisons in all: nothing next to
 * the launch at a decode step's size, and about as long as the copy itself for 16k tokens.
 * Only num_kv_heads, head_dim, block_size, num_blocks and dtype of desc are used.
 */
pkv_status kv_write(const pkv_attn_desc *desc, const void *k_new, const void *v_new,
                    const int64_t *slot_mapping, int32_t num_tokens, void *k_pool,
                    void *v_pool, void *stream);

/*
 * One decode step in one launch: kv_write of each sequence's newest token followed by
 * paged_attn_decode, with the write done inside the decode kernel ("Memory Optimization in
 * LLM Serving with PagedAttention", section "How PagedAttention Works": the new token's
 * K/V goes into its slot, then attention runs over the whole context).  The result equals
 *     kv_write(desc, k_new, v_new, slot_mapping, num_seqs, k_pool, v_pool, stream);
 *     paged_attn_decode(desc, q, k_pool, v_pool, block_tables, context_lens, scale, out,
 *                       workspace, workspace_bytes, stream);
 * bit for bit, under these conditions:
 *   - token s of k_new / v_new ([S, H_kv, D] dtype, 16-byte aligned) belongs to sequence s,
 *     and slot_mapping[s] (int64 [S], 8-byte aligned) is -1 (no write) or the slot of
 *     position context_lens[s]-1, i.e. block_tables[s][(L-1)/B]*B + (L-1)%B;
 *   - the block holding that slot is read by no other sequence of the batch (copy-on-write
 *     of shared blocks, kv_copy_blocks, must already have run; the block manager's
 *     append_slot(s) guarantees this).
 * A slot that is neither -1 nor the slot of position L-1 is not written and sets
 * PKV_FAULT_BAD_SLOT.  Other arguments, errors and the workspace are as paged_attn_decode's.
 * FP8 pools are rejected (PKV_ERR_INVALID).
 */
pkv_status kv_write_and_decode(const pkv_attn_desc *desc, const void *q, const void *k_new,
                               const void *v_new, const int64_t *slot_mapping, void *k_pool,
                               void *v_pool, const int32_t *block_tables,
                               const int32_t *context_lens, float scale, void *out,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode attention over a CONTIGUOUS cache, with no block table: the layout the paged cache
 * replaces, kept as the baseline for the cost of the table ("vLLM and PagedAttention: How
 * Ideas from Operating Systems Accelerated LLM Inference": the paged kernel ran 20-26 %
 * slower than a contiguous one because of the block-table indirection).  Computes exactly
 * what paged_attn_decode computes (same kernel body, same partitions and rounding), with
 * token t of sequence s and kv head h at row t of a reservation of Lmax token rows:
 *   k_cache/v_cache [S, H_kv, Lmax, D] dtype (f16 or bf16), 16-byte aligned, where
 *                   Lmax = desc->max_blocks_per_seq * desc->block_size (rows past
 *                   context_lens[s] are never used)
 *   context_lens    [S] int32, each in [1, Lmax] (checked on the device)
 * q, out, scale, the workspace (pkv_attn_workspace_bytes(desc)) and the errors are as
 * paged_attn_decode's; desc->num_blocks is not used.  S * H_kv * Lmax must stay below 2^31.
 */
pkv_status attn_decode_contiguous(const pkv_attn_desc *desc, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *context_lens, float scale,
                                  void *out, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Copy-on-write block copy ("Memory Optimization in LLM Serving with PagedAttention",
 * section "Advanced Capabilities: Memory Sharing with Copy-on-Write": before a sequence
 * writes into a block it shares, the block's content is copied to a fresh block).  For each
 * pair i, physical block src_dst_pairs[2i+1] of both pools (every kv head and slot) becomes a
 * byte copy of block src_dst_pairs[2i].
 *   src_dst_pairs [num_pairs][2] int32, device memory; destinations distinct and never a
 *                 source of any pair
 * Checked on the device: a pair naming a block outside the pool is skipped
 * (PKV_FAULT_BAD_PAIR); a pair whose destination another pair also names, or that some pair
 * (itself included) reads as its source, is skipped (PKV_FAULT_DUPLICATE).  The remaining
 * pairs are copied, so the result does not depend on the order in which copies run.
 * Only num_kv_heads, head_dim, block_size, num_blocks and dtype of desc are used.
 */
pkv_status kv_copy_blocks(const pkv_attn_desc *desc, const int32_t *src_dst_pairs,
                          int32_t num_pairs, void *k_pool, void *v_pool, void *stream);

/*
 * Swap whole blocks between the device pools and a host pool ("vLLM and PagedAttention: How
 * Ideas from Operating Systems Accelerated LLM Inference": when memory runs short, whole
 * sequences are evicted by swapping them to CPU memory).  host_k / host_v are pinned host
 * buffers of num_host_blocks blocks, [num_host_blocks][H_kv][B][D] dtype each, allocated
 * so the device can reach them (cudaHostAlloc / cudaMallocHost, or torch pin_memory); other
 * host memory is rejected with PKV_ERR_INVALID before any launch.  pairs is device int32
 * [num_pairs][2]:
 *   kv_swap_out: (device block, host block) -- host block := device block, K and V;
 *   kv_swap_in:  (host block, device block) -- device block := host block, K and V.
 * Block ids outside their pool are skipped and set PKV_FAULT_BAD_PAIR; pairs whose
 * destination another pair also names are skipped and set PKV_FAULT_DUPLICATE.  The copies
 * cross PCIe from the kernel itself (one launch per call, whatever the number of blocks).
 * pkv_bm_swap_out / pkv_bm_swap_in produce the pairs.
 */
pkv_status kv_swap_out(const pkv_attn_desc *desc, const int32_t *pairs, int32_t num_pairs,
                       const void *k_pool, const void *v_pool, void *host_k, void *host_v,
                       int32_t num_host_blocks, void *stream);
pkv_status kv_swap_in(const pkv_attn_desc *desc, const int32_t *pairs, int32_t num_pairs,
                      const void *host_k, const void *host_v, int32_t num_host_blocks,
                      void *k_pool, void *v_pool, void *stream);

/*
 * FP8 (E4M3) KV cache ("Memory Optimization in LLM Serving with PagedAttention", section
 * "Broader Context: vLLM, TGI, and TensorRT-LLM": paged KV caches also kept in INT8/FP8).
 * Format (this library's; the page names none):
 *   - k_scale, v_scale: device fp32 [H_kv], each finite and > 0; element x is stored as the
 *     E4M3 code of x / scale (fp32 division, round to nearest even, saturating to +-448)
 *     and means code * scale.  A head whose K or V scale is not finite and > 0 sets
 *     PKV_FAULT_BAD_SCALE: the writes skip that head's values and the decode's output for
 *     its query heads is unspecified;
 *   - k_pool: [NB][H_kv][B][D] bytes;  v_pool: [NB][H_kv][B/16][D][16] bytes: each
 *     16-token half of a block transposed, slot p of a row holding token
 *     2*(p>>2) + (p&1) + 8*((p>>1)&1) of the half (for B = 16 this is [NB][H_kv][D][16]).
 * Only head_dim 128 is built.  Pools are 16-byte aligned.  kv_copy_blocks and kv_swap_* move
 * these blocks with desc->dtype = PKV_FP8_E4M3.
 *
 * kv_write_fp8: desc->dtype is the type of k_new / v_new ([T][H_kv][D]); codes are written
 * into the slots of slot_mapping (-1 skips; others range-checked on the device, and slots
 * named twice skipped, as in kv_write).
 *
 * paged_attn_decode_fp8: as paged_attn_decode, with desc->dtype the type of q and out
 * (PKV_F16 or PKV_BF16); the same workspace rule (pkv_attn_workspace_bytes(desc)).  With
 * desc->partition_tokens 0 it may split contexts more coarsely than the 16-bit decode;
 * pkv_fp8_partition_tokens(desc) reports the partition it uses.
 * Both products run on f16 tensor-core tiles with the K and V codes widened exactly to f16
 * (every E4M3 value is an f16 value) and q rounded to f16 (exact for an f16 q; a bf16 q is
 * first scaled by a power of two, so only values 2^-28 below its row's largest lose bits);
 * accumulation is fp32.  The K scale multiplies the scores and the V scale the output.  Results stay within the q dtype's tolerance of the exact attention over the
 * dequantised codes (2e-3 for f16, 1e-2 for bf16).
 */
/*
 * Partition size, in tokens, that paged_attn_decode_fp8 / kv_write_fp8_and_decode use for
 * this descriptor on the current device: desc->partition_tokens when it is set; otherwise
 * the library's choice, 512, or 2048 when the batch's (sequence, kv head) pairs alone give
 * at least four CTAs per resident CTA slot.  Never needs more workspace than
 * pkv_attn_workspace_bytes(desc).  Returns 0 and sets the last error on an invalid desc.
 * The library's choice depends on the current device's SM count, and the partition changes
 * the rounding order of the result: callers that need the same bits on every GPU model
 * pass an explicit partition_tokens.
 */
int32_t pkv_fp8_partition_tokens(const pkv_attn_desc *desc);

pkv_status kv_write_fp8(const pkv_attn_desc *desc, const void *k_new, const void *v_new,
                        const int64_t *slot_mapping, int32_t num_tokens, const float *k_scale,
                        const float *v_scale, void *k_pool, void *v_pool, void *stream);
pkv_status paged_attn_decode_fp8(const pkv_attn_desc *desc, const void *q, const void *k_pool,
                                 const void *v_pool, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables,
                                 const int32_t *context_lens, float scale, void *out,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * kv_write_fp8 of each sequence's newest token fused into paged_attn_decode_fp8 (one launch),
 * as kv_write_and_decode is for 16-bit pools: token s of k_new / v_new ([S, H_kv, D] of
 * desc->dtype, 16-byte aligned) is quantised into slot_mapping[s] (int64 [S]), which must be
 * -1 or the slot of position context_lens[s]-1 in a block no other sequence of the batch
 * reads.  The pools then hold exactly what kv_write_fp8 writes and the output equals
 * paged_attn_decode_fp8's on those pools, bit for bit.  A slot other than -1 or position
 * L-1's is not written and sets PKV_FAULT_BAD_SLOT.
 */
pkv_status kv_write_fp8_and_decode(const pkv_attn_desc *desc, const void *q, const void *k_new,
                                   const void *v_new, const int64_t *slot_mapping,
                                   const float *k_scale, const float *v_scale, void *k_pool,
                                   void *v_pool, const int32_t *block_tables,
                                   const int32_t *context_lens, float scale, void *out,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Allocation-free variant of paged_attn_decode.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- for example a serving
 * engine that hands (nearly) all free HBM to its KV pool at start-up and owns every later
 * allocation, a plugin or custom-op interface whose host framework forbids allocating inside
 * the op, or a latency-critical loop where cudaMalloc/cudaFree would synchronise the device.
 * It takes the same arguments as paged_attn_decode minus the workspace, and keeps the
 * split-context partial results in a scratch array that is part of the library itself:
 * PKV_STATIC_WORKSPACE_BYTES of device memory, held on every GPU that loads the library
 * until the process exits.  It calls no allocating routine.
 *   - The first call on a device looks up that device's copy of the array (once per
 *     device, with that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset (or anything
 *     else that destroys the device's primary context) it is stale, and this entry point
 *     must not be called again in that process.
 *   - A batch whose split scratch (pkv_attn_workspace_bytes) exceeds
 *     PKV_STATIC_WORKSPACE_BYTES is rejected with PKV_ERR_INVALID; nothing is launched.
 *   - Every call on a device shares the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero: each partial is written before it is read).
 *     Calls whose work overlaps on the GPU (other streams, other host threads) race on it:
 *     order them on one stream, or use paged_attn_decode with a workspace per stream.
 */
#define PKV_STATIC_WORKSPACE_BYTES (32u << 20)
pkv_status paged_attn_decode_no_alloc(const pkv_attn_desc *desc, const void *q,
                                      const void *k_pool, const void *v_pool,
                                      const int32_t *block_tables,
                                      const int32_t *context_lens, float scale, void *out,
                                      void *stream);

/*
 * Read the device fault word of the current device into *faults (host) after the work
 * queued on stream so far has finished; clear != 0 resets it to 0.  Synchronises stream.
 */
pkv_status pkv_device_faults(uint32_t *faults, int clear, void *stream);

/* ---------------------------------------------------------------------------------------
 * Host block manager ("Memory Optimization in LLM Serving with PagedAttention", sections
 * "How PagedAttention Works" (on-demand allocation, fragmentation only in the last block)
 * and "Advanced Capabilities: Memory Sharing with Copy-on-Write" (shared blocks, reference
 * counts, copy before write); "vLLM and PagedAttention: How Ideas from Operating Systems
 * Accelerated LLM Inference" (16-token blocks, fork-style sharing for parallel sampling)).
 *
 * Host only: it hands out block ids and slots and never touches device memory.  Sequence
 * ids are caller-chosen int64.  The free list is first-in first-out (allocation takes its
 * head, a block whose reference count drops to 0 joins its tail).  A call that fails with
 * PKV_ERR_OOM changes nothing.  Not thread-safe: one thread per manager at a time.
 * ------------------------------------------------------------------------------------- */
typedef struct pkv_bm pkv_bm;

/* initial_free_order: host [num_blocks] permutation of 0..num_blocks-1, or NULL for
 * ascending order.  block_size is 16 or 32. */
pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size,
                         const int32_t *initial_free_order, pkv_bm **out);
void pkv_bm_destroy(pkv_bm *bm);

/* Register sequence seq holding num_tokens tokens (a prompt): ceil(num_tokens/block_size)
 * fresh blocks, all or nothing. */
pkv_status pkv_bm_add_seq(pkv_bm *bm, int64_t seq, int32_t num_tokens);

/* Give the next token of seq a slot.  If the token opens a new block, a fresh block is
 * appended.  Otherwise, if the last block is shared (reference count > 1), a fresh block dst
 * replaces it in seq's table, the old block's count drops by one, and (*cow_src, *cow_dst)
 * = (old, dst) tells the caller to run kv_copy_blocks before writing; else both are -1. */
pkv_status pkv_bm_append_slot(pkv_bm *bm, int64_t seq, int64_t *slot_out, int32_t *cow_src,
                              int32_t *cow_dst);

/* append_slot for n sequences in order, all or nothing.  slots_out [n] int64 (host);
 * cow_pairs_out [n][2] int32 (host) receives *num_cow pairs. */
pkv_status pkv_bm_append_slots(pkv_bm *bm, const int64_t *seqs, int32_t n,
                               int64_t *slots_out, int32_t *cow_pairs_out,
                               int32_t *num_cow);

/* child maps the same physical blocks as parent (every count + 1) and has its length. */
pkv_status pkv_bm_fork(pkv_bm *bm, int64_t parent, int64_t child);

/* Drop seq; blocks whose count reaches 0 return to the free list in table order. */
pkv_status pkv_bm_free_seq(pkv_bm *bm, int64_t seq);

/* Copy seq's block table into out (host, capacity cap); *n = its length (also when
 * cap < *n, in which case PKV_ERR_INVALID is returned and out holds the first cap). */
pkv_status pkv_bm_block_table(const pkv_bm *bm, int64_t seq, int32_t *out, int32_t cap,
                              int32_t *n);

/* Pack the tables of n sequences into out [n][max_blocks] (host, -1 padded) and their
 * lengths into lens_out [n] (host). */
pkv_status pkv_bm_block_tables(const pkv_bm *bm, const int64_t *seqs, int32_t n,
                               int32_t max_blocks, int32_t *out, int32_t *lens_out);

pkv_status pkv_bm_seq_len(const pkv_bm *bm, int64_t seq, int32_t *len);
pkv_status pkv_bm_refcount(const pkv_bm *bm, int32_t block, int32_t *count);
int32_t pkv_bm_num_free(const pkv_bm *bm);
int32_t pkv_bm_num_seqs(const pkv_bm *bm);

/* Copy the free list, head first, into out (host, capacity cap); returns its length. */
int32_t pkv_bm_free_list(const pkv_bm *bm, int32_t *out, int32_t cap);

/* Host (swap) pool of num_host_blocks blocks with its own first-in first-out free list
 * (initial_free_order: permutation or NULL = ascending).  Host blocks each hold one swapped
 * sequence's data and are never shared.  Fails while any sequence is swapped out. */
pkv_status pkv_bm_set_host_pool(pkv_bm *bm, int32_t num_host_blocks,
                                const int32_t *initial_free_order);

/* Evict seq to the host pool: each table entry j gets a fresh host block h_j and
 * pairs_out[j] = (device block, h_j) (host, capacity cap pairs; *n = table length).  The
 * device block loses one reference and returns to the free list when none is left, so run
 * kv_swap_out on these pairs before any later write can reuse it.  All or nothing
 * (PKV_ERR_OOM when the host pool is short).  A swapped-out sequence can only be swapped
 * in or freed. */
pkv_status pkv_bm_swap_out(pkv_bm *bm, int64_t seq, int32_t *pairs_out, int32_t cap,
                           int32_t *n);

/* Bring seq back: each host block gets a fresh device block, pairs_out[j] = (host block,
 * device block); the host blocks return to the host free list.  All or nothing.  Blocks
 * that were shared before the swap come back as private copies. */
pkv_status pkv_bm_swap_in(pkv_bm *bm, int64_t seq, int32_t *pairs_out, int32_t cap,
                          int32_t *n);

pkv_status pkv_bm_is_swapped(const pkv_bm *bm, int64_t seq, int32_t *swapped);
int32_t pkv_bm_num_host_free(const pkv_bm *bm);

/* ---- measurement aid -------------------------------------------------------------------- */
/*
 * Read-bandwidth probe (the pages have no counterpart: it gives the roofline a read-only
 * denominator).  Streams chunk_bytes-sized chunks of the device buffer buf into shared
 * memory with 1-D bulk copies, in a fixed scattered order (a bijective hash of the chunk
 * index), and discards them; n is the largest power of two with n * chunk_bytes <= bytes.  Every chunk
 * is read once; nothing is written.  Time it with events on the stream.
 *   buf: device pointer, 16-byte aligned, owned by the caller;
 *   chunk_bytes: 2048, 4096, 8192 or 16384;
 *   ctas_per_sm: CTAs of 2 warps (4 copies in flight each) launched per SM; 0 = as many as
 *     fit; more than fit run in turns;
 *   bytes_read: host out (may be NULL) = n * chunk_bytes.
 * Errors: PKV_ERR_INVALID for a null or unaligned buf, an unsupported chunk, fewer than one
 * chunk or more than 2^31 chunks, a negative ctas_per_sm; PKV_ERR_CUDA for a failed launch.  A copy wait that runs
 * out sets PKV_FAULT_TIMEOUT in the device fault word.
 */
pkv_status pkv_read_probe(const void *buf, size_t bytes, int32_t chunk_bytes,
                          int32_t ctas_per_sm, size_t *bytes_read, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
