/*
 * libtaco_attn: paged tree-attention verify and paged KV-append for NVIDIA B200 (sm_100a).
 *
 * The operations come from public TACO-LLM pages:
 *  - paging: "大模型倍速推理引擎 TACO-LLM 的设计与实践" (53ai.com workshop page), section
 *    "4. 支持 Paged Attention": a sequence's KV cache is cut into blocks of a fixed number of tokens,
 *    and consecutive logical blocks map to non-contiguous physical blocks through a block table;
 *    blocks are filled as new tokens are produced.
 *  - verification and tree attention: same page, sections "TACO-LLM 如何解决大模型推理瓶颈?",
 *    "优化方案设计思路" and "优化策略总结" item 1: the target model checks a batch of candidate tokens
 *    in one parallel pass, and candidates sharing a prefix share its computation (each candidate sees
 *    the committed prefix and its own ancestors).
 *  - TurboAttention: same page, the kernel bullets under "整体方案分为两大部分" (paged + flash-style
 *    fused softmax; several candidates turn vector-matrix into matrix-matrix work for tensor cores),
 *    and the 618zxw.cn article, section "長シーケンス推論最適化におけるTurboAttention".
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device, owned by the caller, and must
 *    stay valid until the work enqueued on `stream` has finished. Nothing is copied to or from host.
 *  - Calls only enqueue work on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *    return; they do not synchronise.
 *  - Every array is dense, row-major, innermost dimension last. 16-bit float tensors must start on a
 *    16-byte boundary.
 *  - Host-side validation runs before any launch; a non-OK status means nothing was enqueued, and
 *    taco_attn_last_error() gives a message (thread-local).
 *  - Values inside device arrays (block ids, lengths, slots) are checked on the device: an
 *    out-of-range value sets a bit in an error word and the offending access is skipped (it never
 *    faults or traps). Each (device, stream) pair has its own word; taco_attn_check_device(stream)
 *    reads and clears the word of the current device and that stream.
 *  - Library-owned device memory (the error word and the split-KV workspace) is kept per (device,
 *    stream handle). Calls on different streams may therefore run concurrently; calls on one stream
 *    are ordered by the stream. A stream handle that is destroyed while its work is still queued and
 *    then reused by a new stream shares the old workspace: let such work finish first.
 *    paged_tree_attention_noalloc is the exception: it uses one fixed array per device (see there).
 *
 * Shapes: B batch, C max candidates per sequence (1..32), Hq / Hkv query / KV heads (Hq % Hkv == 0,
 * G = Hq / Hkv), D head dim (64 or 128), bs block size (power of two, 8..256), NB physical blocks,
 * maxblk block-table columns.
 */
#ifndef TACO_ATTN_H
#define TACO_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t taco_status;
#define TACO_OK 0
#define TACO_ERR_INVALID_ARG 1   /* null pointer, bad size, misaligned pointer */
#define TACO_ERR_UNSUPPORTED 2   /* a size the library has no kernel for (D, bs, C) */
#define TACO_ERR_CUDA 3          /* a CUDA runtime call or launch failed */
#define TACO_ERR_DEVICE_CHECK 4  /* taco_attn_check_device found a device-side range error */

#define TACO_DTYPE_F16 0
#define TACO_DTYPE_BF16 1

/* Device error word bits (taco_attn_check_device). */
#define TACO_DEVERR_BLOCK_ID 0x1u       /* block table entry outside [0, NB) */
#define TACO_DEVERR_CONTEXT_LEN 0x2u    /* context_lens[b] outside [0, maxblk * bs] */
#define TACO_DEVERR_NUM_CAND 0x4u       /* num_candidates[b] outside [0, min(C, context_lens[b])] */
#define TACO_DEVERR_SLOT 0x8u           /* slot_offsets[b][i] >= maxblk * bs */
#define TACO_DEVERR_WAIT_TIMEOUT 0x10u  /* a pipeline wait gave up (the kernel returned early) */
#define TACO_DEVERR_PARENT 0x20u        /* parents[b][i] outside [-1, i) */
#define TACO_DEVERR_TABLE_FULL 0x40u    /* prefix_cache_insert probed every slot without a place */

/*
 * paged_tree_attention: masked softmax attention of every candidate query over its sequence's
 * paged keys (the TurboAttention verify pass).
 *
 *   q               [B, C, Hq, D]   dtype; row (b, i, h) is candidate i of sequence b, query head h
 *   k_cache,v_cache [NB, Hkv, bs, D] dtype; (block, kv head, slot, dim)
 *   block_tables    int32 [B, maxblk]; logical block j of sequence b is physical block
 *                   block_tables[b*maxblk + j] (entries past ceil(L_b/bs) are never read)
 *   context_lens    int32 [B]; L_b = number of keys of sequence b, its n_b candidates included; the
 *                   candidates' K/V sit at logical positions P_b .. L_b-1, P_b = L_b - n_b (written
 *                   before this call, e.g. by paged_kv_append)
 *   num_candidates  int32 [B]; n_b, 0 <= n_b <= min(C, L_b)
 *   tree_mask_bits  uint32 [B, C]; bit j of word (b, i): candidate i may attend to candidate j.
 *                   Bits j >= n_b are ignored. Any pattern is allowed (a chain is 2^(i+1)-1, a tree
 *                   is the ancestor-or-self set).
 *   scale           multiplies q.k before the softmax (usually 1/sqrt(D))
 *   out             [B, C, Hq, D] dtype, written completely: row (b, i, h) with i < n_b is
 *                   sum_p softmax_p(scale q.k_p) v_p over the visible positions p (the prefix
 *                   0..P_b-1 plus the candidates its mask word selects); rows i >= n_b and rows that
 *                   see no key are zeros. Must not alias any input.
 *   query head h reads KV head h / G.
 * Softmax state (max, sum) and the output accumulator are fp32; the result is rounded once to
 * `dtype` (round to nearest even). The library keeps a workspace for split-KV partial results per
 * (device, stream); the first call on a stream (or one that needs a larger workspace) allocates it
 * with cudaMalloc and therefore synchronises the device. Calls on different streams use different
 * workspaces and may overlap on the GPU.
 * Kernels: one verify launch; when a call has few work units against the grid (a handful of long
 * sequences, whose units are then cut into many split-KV pieces), a second, separate combine kernel
 * merges the pieces (TACO_OPT_COMBINE; taco_attn_last_call_launches reports what a call enqueued).
 */
taco_status paged_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                 float scale, void* out,
                                 int32_t dtype, int32_t batch, int32_t max_candidates,
                                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                 void* stream);

/*
 * paged_kv_append: write the candidates' new K/V rows into their cache slots through the block
 * table (paging section cited above: blocks are filled as tokens are generated).
 *
 *   k_new, v_new    [B, C, Hkv, D] dtype
 *   block_tables    int32 [B, maxblk]
 *   slot_offsets    int32 [B, C]; logical position s of row (b, i); s < 0 means "skip this row".
 *                   Row (b, i, h) is copied bit-for-bit to cache[block_tables[b][s / bs], h, s % bs, :].
 *                   Slots within one call must be distinct (otherwise which row lands is undefined).
 *   k_cache,v_cache [NB, Hkv, bs, D] dtype, updated in place; no other byte changes.
 */
taco_status paged_kv_append(const void* k_new, const void* v_new, const int32_t* block_tables,
                            const int32_t* slot_offsets, void* k_cache, void* v_cache,
                            int32_t dtype, int32_t batch, int32_t max_candidates,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t num_blocks, int32_t max_blocks_per_seq, void* stream);

/*
 * paged_tree_attention_append: paged_kv_append of the candidates followed by paged_tree_attention, in one
 * call. Candidate i < n_b of sequence b goes to logical slot P_b + i (P_b = L_b - n_b; the layout
 * paged_tree_attention assumes), so no slot array is needed; the caches are updated exactly as
 * paged_kv_append would update them and `out` equals paged_tree_attention's result on the updated
 * caches.
 *   k_new, v_new  [B, C, Hkv, D] dtype, 16-byte aligned; rows i >= n_b are not read.
 * Units of at most 16 packed query rows run the append inside the verify kernel: the CTA that loads the
 * tile holding a candidate's key puts the new row into its shared-memory copy and into the cache, so no
 * separate launch is needed. Other shapes launch the append kernel first on the same stream.
 * Slot block ids outside [0, NB) are skipped and flagged (TACO_DEVERR_BLOCK_ID).
 */
taco_status paged_tree_attention_append(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                        void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                                        const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                        float scale, void* out,
                                        int32_t dtype, int32_t batch, int32_t max_candidates,
                                        int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                        void* stream);

/*
 * paged_tree_attention_noalloc: the same arguments and result (within the tolerance that holds for
 * every kernel of this library) as paged_tree_attention, for callers that cannot allocate device
 * memory. The pages have no counterpart of this entry point;
 * it exists because paged_tree_attention grows a workspace with cudaMalloc on first use, which a
 * caller cannot allow when it runs under a fixed memory-pool budget (e.g. a server that has handed
 * all free HBM to its KV cache), when an implicit device synchronisation mid-step is not acceptable,
 * or when allocation after start-up is forbidden.
 *   - Scratch: a fixed 24 MiB array inside the library's device image (every GPU that loads the
 *     library holds it until exit); no cudaMalloc, cudaFree or other allocating call is made.
 *   - Limit: at most 65536 work units (batch * num_kv_heads * row groups); larger calls return
 *     TACO_ERR_UNSUPPORTED with a message and enqueue nothing. The grid is capped so that the split-KV
 *     partials fit the scratch, which holds both kernels' full grids on a 148-SM B200.
 *   - Kernel: the one paged_tree_attention picks by itself for 16-bit caches (tcgen05 for
 *     G * C >= 48, mma.sync otherwise); TACO_OPT_KERNEL and TACO_OPT_GRID_CTAS do not apply. Measured
 *     on B200 it takes 0.99-1.01x the time of paged_tree_attention on the bench's four workloads.
 *   - All calls on a device share the array and it keeps the last call's contents; each call clears
 *     what must start at zero on `stream` first. Calls whose work overlaps on the GPU race: order them
 *     on one stream.
 *   - The first call on a device (of this function or of taco_attn_check_noalloc) looks up the
 *     array's address (cudaGetSymbolAddress, that device current); make it before any stream capture.
 *   - Device-side range violations and wait timeouts are skipped and recorded in the array's own
 *     error word, which accumulates until taco_attn_check_noalloc reads and clears it.
 */
taco_status paged_tree_attention_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, const int32_t* context_lens,
                                         const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                         float scale, void* out,
                                         int32_t dtype, int32_t batch, int32_t max_candidates,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                         void* stream);

/*
 * taco_attn_check_noalloc: synchronise `stream`, then read and clear the error word of
 * paged_tree_attention_noalloc's fixed array on the current device (TACO_DEVERR_* bits). Returns
 * TACO_OK if it was zero, TACO_ERR_DEVICE_CHECK otherwise (bits in the message and in *bits_out when
 * bits_out is not NULL). Allocates nothing. The pages have no counterpart of this function: it only
 * reports the errors of the allocation-free entry point above.
 */
taco_status taco_attn_check_noalloc(void* stream, uint32_t* bits_out);

/*
 * 8-bit KV cache. The 53ai.com workshop page (section "5. 支持 Quantization（模型量化）") lists 8-bit
 * (INT8 / FP8) storage among the engine's features for its lower memory and bandwidth needs, the
 * 618zxw.cn page (section "LLM量子化技術による推論コストの削減") has quantised attention operators with
 * fast dequantisation, and the 17173xz.com overview counts quantised operators among its kernels; none
 * fixes a format. These calls use e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; 0x7F / 0xFF are NaN; largest finite 448) with one float32 scale per KV head for K and
 * one for V:
 *   stored code  = e4m3(x / scale[h])  (float32 quotient correctly rounded, then the nearest e4m3 value,
 *                  ties to the even code, magnitudes above 448 saturate to 448, NaN stays NaN)
 *   value read   = decode(code) * scale[h]
 * The cache layout is [NB, Hkv, bs, D] with one byte per element.
 *
 * paged_kv_append_e4m3: paged_kv_append into e4m3 caches. k_new / v_new are [B, C, Hkv, D] `dtype`
 * (F16 / BF16); k_scale, v_scale are device float32 [Hkv] (finite and nonzero: not checked). Every
 * other argument and rule is that of paged_kv_append; D is 64 or 128.
 */
taco_status paged_kv_append_e4m3(const void* k_new, const void* v_new, const int32_t* block_tables,
                                 const int32_t* slot_offsets, const float* k_scale, const float* v_scale,
                                 void* k_cache, void* v_cache, int32_t dtype, int32_t batch,
                                 int32_t max_candidates, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                 void* stream);

/*
 * paged_tree_attention_e4m3: paged_tree_attention over e4m3 caches (layout and scales as above): the
 * result is that of paged_tree_attention with K = decode(k_cache) * k_scale[h] and V = decode(v_cache) *
 * v_scale[h]. q and out are `dtype` (F16 / BF16). Every size paged_tree_attention takes is supported
 * (head_dim 64 or 128, any packed query rows). Narrow tiles (head_dim 128, fewer than 48 packed rows)
 * run a warp-MMA kernel that widens the codes in registers; every other shape runs the tensor-core
 * (tcgen05) kernel, which widens each tile of codes once, exactly, to f16 in shared memory. For bf16
 * queries that kernel multiplies each query row by a power of two and rounds it to f16 (exact for every
 * element down to 2^-29 of the row's largest magnitude) in the workspace first. The workspace rules of
 * paged_tree_attention apply. k_scale, v_scale: device float32 [Hkv], finite and nonzero (not checked).
 */
taco_status paged_tree_attention_e4m3(const void* q, const void* k_cache, const void* v_cache,
                                      const float* k_scale, const float* v_scale,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                      float scale, void* out,
                                      int32_t dtype, int32_t batch, int32_t max_candidates,
                                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                      void* stream);

/*
 * paged_tree_attention_append_e4m3: paged_kv_append_e4m3 of each sequence's candidates into logical
 * slots P_b .. L_b - 1 (slot_offsets derived as for paged_tree_attention_append), then
 * paged_tree_attention_e4m3 over the updated caches, in one call. k_new, v_new: [B, C, Hkv, D] `dtype`.
 * On the mma.sync kernel (head_dim 128) with units of at most 16 packed query rows, the verify kernel
 * quantises the candidates' rows itself: the CTA that loads the tile holding a candidate's key divides
 * each new value by its head's scale and rounds it to e4m3 exactly as paged_kv_append_e4m3 does, then
 * writes the codes into its shared-memory copy of the tile and into the cache. One launch, no append
 * kernel. Otherwise the quantising append kernel runs first on `stream`. The verify then reads all
 * but the appended slots before the append ends, unless a query conversion runs in between (bf16
 * queries on the tcgen05 kernel). Every other argument, rule and error is that of the two calls.
 */
taco_status paged_tree_attention_append_e4m3(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                             void* v_cache, const float* k_scale, const float* v_scale,
                                             const int32_t* block_tables, const int32_t* context_lens,
                                             const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                             float scale, void* out, int32_t dtype, int32_t batch,
                                             int32_t max_candidates, int32_t num_q_heads, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                             int32_t max_blocks_per_seq, void* stream);

/*
 * The step after the verify. The pages ("大模型倍速推理引擎 TACO-LLM 的设计与实践", sections
 * "TACO-LLM 如何解决大模型推理瓶颈?", "优化方案设计思路" and "优化策略总结") have the target model
 * validate candidate tokens obtained ahead of time, organised as a forest (multi-branch prediction),
 * and count the candidates' hit length; they fix no acceptance rule. These calls implement the plain
 * greedy one:
 *  - candidate i is correct iff its token equals the target's argmax after its parent (after the
 *    committed prefix for a root);
 *  - a candidate is accepted iff it and all its ancestors are correct; the hit is the deepest accepted
 *    candidate (the smallest index among equally deep ones) and the accepted path runs from its root
 *    to it;
 *  - the target's argmax after the hit (after the prefix when nothing is accepted) is one more token
 *    the step emits (the bonus token);
 *  - the accepted candidates' K/V move to the contiguous tail: the path's d-th node (0-based) goes to
 *    logical slot P_b + d, P_b = L_b - n_b. Passing slot_offsets_out with the step's k_new / v_new to
 *    paged_kv_append performs that move.
 *
 * tree_mask_from_parents: the tree_mask_bits of paged_tree_attention from parent links.
 *   parents         int32 [B, C]; parents[b][i] = -1 (a root) or a candidate j < i
 *   num_candidates  int32 [B]; n_b in [0, C]
 *   mask_out        uint32 [B, C]; bit j of word (b, i) is set iff j is i or an ancestor of i; rows
 *                   i >= n_b are 0
 * C in 1..32. A parent outside [-1, i) sets TACO_DEVERR_PARENT and ends that row's walk.
 */
taco_status tree_mask_from_parents(const int32_t* parents, const int32_t* num_candidates, int32_t batch,
                                   int32_t max_candidates, uint32_t* mask_out, void* stream);

/*
 * logits_argmax: per row of a [rows, vocab] matrix of 16-bit floats, the smallest index of the largest
 * value. NaN never wins; a row without a number above -inf gives 0.
 *   logits     [rows, vocab] dtype (TACO_DTYPE_F16 / TACO_DTYPE_BF16), dense
 *   out_index  int32 [rows]
 * rows >= 0, vocab >= 1. The pointer need not be 16-byte aligned (a slower kernel reads it then).
 */
taco_status logits_argmax(const void* logits, int32_t dtype, int64_t rows, int32_t vocab, int32_t* out_index,
                          void* stream);

/*
 * tree_greedy_accept: acceptance of each sequence's candidate forest (rules above).
 *   target_argmax     int32 [B, C + 1]; row 0: the target's argmax after the prefix, row i + 1: after
 *                     candidate i (e.g. logits_argmax over [B, C + 1, vocab] logits)
 *   candidate_tokens  int32 [B, C]
 *   parents           int32 [B, C]; -1 or an earlier candidate
 *   num_candidates    int32 [B]; n_b in [0, min(C, L_b)]
 *   context_lens      int32 [B]; L_b as in paged_tree_attention (candidates included)
 *   accept_len        int32 [B]; length of the accepted path (0..n_b)
 *   accepted_path     int32 [B, C]; its nodes root first, -1 after accept_len
 *   bonus_token       int32 [B]
 *   slot_offsets_out  int32 [B, C]; P_b + d for the path's d-th node, -1 for every other candidate
 * C in 1..32. Parents outside [-1, i) set TACO_DEVERR_PARENT (that candidate is treated as an
 * incorrect root); n_b out of range sets TACO_DEVERR_NUM_CAND and is clamped.
 */
taco_status tree_greedy_accept(const int32_t* target_argmax, const int32_t* candidate_tokens,
                               const int32_t* parents, const int32_t* num_candidates, const int32_t* context_lens,
                               int32_t batch, int32_t max_candidates, int32_t* accept_len, int32_t* accepted_path,
                               int32_t* bonus_token, int32_t* slot_offsets_out, void* stream);

/*
 * Prefix-tree KV lookup for prefill. The 618zxw.cn page (section "プレフィックスキャッシュ技術を使用して
 * TTFTを削減する"), the 17173xz.com overview's prefill paragraph and the tencentcloud.com document's list
 * of techniques keep earlier requests' prefill KV in a prefix tree, so that prefill becomes a lookup of
 * cached KV and only the tokens not found are computed. Here a node is one full KV block of block_size
 * tokens, identified by the whole token prefix it ends; it owns the physical block holding that
 * prefix's K/V. A partial trailing block is never cached or matched.
 *
 * The tree lives in caller-owned device memory:
 *   slot_keys    uint64 [capacity]  open-addressing table of node keys, 8-byte aligned; 0 = empty.
 *                                   Set every entry to 0 once before the first insert.
 *   slot_nodes   int32  [capacity]  node (physical block) of each claimed slot; set every entry to -1
 *                                   once, together with slot_keys.
 *   node_parent  int32  [NB]        node of the prefix one block shorter, -1 for a first block
 *   node_depth   int32  [NB]        the node's block index within its sequence (0 = first block)
 *   node_tokens  int32  [NB, block_size]  the node's tokens
 * capacity is a power of two; keep it at least twice the number of nodes (probe chains stay short).
 * A key is a 64-bit hash of the whole prefix; every match is confirmed on depth, parent and tokens, so a
 * hash collision never changes a result. Inserts and lookups that overlap on the GPU race: order them.
 *
 * Sequences (both calls): tokens int32 [total]; sequence b is tokens[seq_starts[b] .. seq_starts[b+1])
 * (seq_starts int32 [batch + 1], non-decreasing: a decreasing pair sets TACO_DEVERR_CONTEXT_LEN and
 * counts as empty). Only the first min(len_b / block_size, max_blocks_per_seq) full blocks are used.
 *
 * prefix_cache_lookup: per sequence, the longest run of its leading full blocks whose path is in the
 *   tree. out_blocks int32 [batch, max_blocks_per_seq]: the path's physical blocks (a block-table
 *   prefix), then -1; out_matched int32 [batch]: the run's length in blocks (matched tokens = that
 *   times block_size).
 *
 * prefix_cache_insert: add the full blocks of each sequence, whose K/V sit in block_tables int32
 *   [batch, max_blocks_per_seq] (entries in [0, NB)). A block whose prefix is already a node keeps that
 *   node; otherwise the sequence's own block becomes the node (its node_* entries are written). When
 *   several sequences of one call add the same new prefix, one of their blocks becomes the node (which
 *   one is not fixed) and all of them get it. out_blocks [batch, max_blocks_per_seq]: per full block,
 *   the physical block that holds its prefix afterwards (blocks that did not become nodes can be
 *   freed), then -1. out_inserted int32 [batch] (may be NULL): blocks processed per sequence. A block
 *   id outside [0, NB) sets TACO_DEVERR_BLOCK_ID, and a table with no free slot on the chain sets
 *   TACO_DEVERR_TABLE_FULL; either ends that sequence's walk. A bounded wait for another sequence's
 *   node that times out sets TACO_DEVERR_WAIT_TIMEOUT. A block id that is already a node must not be
 *   passed for a block whose prefix is new.
 */
/*
 * Batched Lookahead Cache (53ai.com workshop page, "整体方案分为两大部分", item 1 "基于批处理的 Lookahead
 * Cache" and the paragraphs after it: candidates for a whole batch from a per-sequence local cache and a
 * shared global cache, queried by match length, a copied length adapted to batch size and hit rate, and
 * a forest of branches).
 *
 * lookahead_propose: a candidate forest per sequence, ready for tree_mask_from_parents and the verify.
 *   history        int32 [total]; sequence b's tokens (prompt plus generated) are
 *                  history[hist_starts[b] .. hist_starts[b+1]), token ids >= 0 (the local cache)
 *   hist_starts    int32 [batch + 1], non-decreasing (a decreasing pair sets TACO_DEVERR_CONTEXT_LEN
 *                  and counts as empty)
 *   global_tokens  int32 [global_len] shared by the batch (the global cache); values < 0 separate
 *                  passages and never match. May be NULL when global_len is 0.
 *   copy_len       int32 [batch]: at most this many tokens are copied per branch (<= 0: no candidates)
 *   max_match      longest context matched, 1..16
 *   Per cache: the longest m <= min(max_match, len_b) such that the sequence's last m tokens occur in
 *   the cache ending at a position e with a following token (local: an earlier occurrence); the
 *   occurrences of that m, most recent (largest e) first, each give the following tokens (at most
 *   copy_len, stopping before a separator or the end) as a path. Local paths, then global ones, merge
 *   into a trie of at most max_candidates (<= 32) nodes numbered in creation order (a parent precedes
 *   its children); merging stops when the trie is full.
 *   tokens_out, parents_out  int32 [batch, max_candidates]: node token and parent (-1 = root); -1 past
 *                  the node count. num_candidates_out int32 [batch].
 *
 * lookahead_update_copy_len: after a verify step, per sequence
 *   hit[b] <- (1 - alpha) * hit[b] + alpha * accept_len[b] / max(1, num_proposed[b])
 *   copy_len[b] = clamp(floor(copy_max * hit[b] * min(1, batch_ref / batch) + 0.5), 1, copy_max)
 *   each operation rounded to float32 in this order. hit float32 [batch] is updated in place.
 */
taco_status lookahead_propose(const int32_t* history, const int32_t* hist_starts, const int32_t* global_tokens,
                              int64_t global_len, const int32_t* copy_len, int32_t max_match, int32_t batch,
                              int32_t max_candidates, int32_t* tokens_out, int32_t* parents_out,
                              int32_t* num_candidates_out, void* stream);

taco_status lookahead_update_copy_len(const int32_t* accept_len, const int32_t* num_proposed, float* hit,
                                      int32_t* copy_len, int32_t batch, int32_t copy_max, float alpha,
                                      int32_t batch_ref, void* stream);

taco_status prefix_cache_lookup(const int32_t* tokens, const int32_t* seq_starts, const uint64_t* slot_keys,
                                const int32_t* slot_nodes, int64_t capacity, const int32_t* node_parent,
                                const int32_t* node_depth, const int32_t* node_tokens, int32_t* out_blocks,
                                int32_t* out_matched, int32_t batch, int32_t block_size, int32_t num_blocks,
                                int32_t max_blocks_per_seq, void* stream);

taco_status prefix_cache_insert(const int32_t* tokens, const int32_t* seq_starts, const int32_t* block_tables,
                                uint64_t* slot_keys, int32_t* slot_nodes, int64_t capacity, int32_t* node_parent,
                                int32_t* node_depth, int32_t* node_tokens, int32_t* out_blocks,
                                int32_t* out_inserted, int32_t batch, int32_t block_size, int32_t num_blocks,
                                int32_t max_blocks_per_seq, void* stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* taco_attn_last_error(void);

/*
 * Synchronise `stream`, then read and clear the error word of (the current device, `stream`): the
 * bits set by calls enqueued on that stream, and by no other stream's calls. Returns TACO_OK if it
 * was zero, TACO_ERR_DEVICE_CHECK otherwise (the bits are in the message and in *bits_out when
 * bits_out is not NULL). After a wait timeout it also clears that stream's split-KV arrival
 * counters. paged_tree_attention_noalloc has its own word: taco_attn_check_noalloc reads it.
 */
taco_status taco_attn_check_device(void* stream, uint32_t* bits_out);

/* Free every (device, stream) workspace (call only when no work using them is in flight). */
void taco_attn_release_workspace(void);

/* Tuning / test knobs (process-wide). */
#define TACO_OPT_GRID_CTAS 1   /* verify grid size in CTAs; 0 = automatic (2 per SM). */
#define TACO_OPT_KERNEL 2      /* 0 = automatic, 1 = mma.sync path, 2 = tcgen05 path (where built) */
#define TACO_OPT_L2_PREFETCH 3 /* key tiles of K/V the verify asks L2 to fetch ahead of its shared-memory
                                  loads: -1 = the kernel's default, 0 = none, up to 64 */
#define TACO_OPT_SEG_COST 5    /* work split of the verify: key tiles each (sequence, KV head, row group)
                                  unit counts on top of its own, for the cost of starting and finishing
                                  it, when the units' tiles are divided between CTAs: -1 = the kernel's
                                  default, 0 = an equal split of the tiles, up to 64 */
#define TACO_OPT_TEST_STALL 4  /* test knob for the bounded pipeline waits, mma.sync verify kernel only:
                                  0 = off (default); t + 1 = the first CTA's producers never arm the
                                  stage of its tile t, so that a consumer's wait runs out after 20 ms,
                                  the call reports TACO_DEVERR_WAIT_TIMEOUT and its output is undefined */
#define TACO_OPT_COMBINE 6     /* split-KV combine: 0 = automatic (mma.sync verify: a separate combine
                                  kernel when the call has at most a quarter as many work units as
                                  CTAs, so that units are cut into many pieces; tcgen05 verify: inside),
                                  1 = inside the verify, by the last CTA to finish each unit, 2 = the
                                  separate kernel for either verify */
taco_status taco_attn_set_option(int32_t key, int64_t value);

/* Kernels the calling thread's last attention call (paged_tree_attention, _append, _e4m3,
 * _append_e4m3) enqueued: the append or query conversion when it ran, the verify, and the combine when
 * it ran separately. 0 when that call failed before its first launch. */
int32_t taco_attn_last_call_launches(void);

/* ABI version of this header (bumped on any signature change). */
int32_t taco_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TACO_ATTN_H */
