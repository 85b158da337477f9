// Internal launcher interface between the host C-ABI (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "taco_attn.h"

namespace taco {

struct VerifyParams;

struct AppendArgs {
  const void* k_new;
  const void* v_new;
  const int32_t* block_tables;
  const int32_t* slot_offsets;
  void* k_cache;
  void* v_cache;
  uint32_t* error_word;
  int B, C, Hkv, D, bs, num_blocks, max_blocks;
  int dtype;  // of k_new / v_new (the quantising append converts them)
  // with slot_offsets null: candidate i < n_b goes to logical slot L_b - n_b + i (the verify's layout)
  const int32_t* context_lens;
  const int32_t* num_candidates;
};

struct MaskArgs {
  const int32_t* parents;
  const int32_t* num_candidates;
  uint32_t* mask_out;
  uint32_t* error_word;
  int B, C;
};

struct AcceptArgs {
  const int32_t* target_argmax;
  const int32_t* tokens;
  const int32_t* parents;
  const int32_t* num_candidates;
  const int32_t* context_lens;
  int32_t* accept_len;
  int32_t* accepted_path;
  int32_t* bonus_token;
  int32_t* slot_offsets_out;
  uint32_t* error_word;
  int B, C;
};

cudaError_t launch_tree_masks(const MaskArgs& a, cudaStream_t stream);
cudaError_t launch_argmax(const void* logits, int dtype, int64_t rows, int vocab, int32_t* out, cudaStream_t stream);
cudaError_t launch_accept(const AcceptArgs& a, cudaStream_t stream);

// Rows of packed queries one unit of the mma.sync verify kernel covers for a given G * C.
int mma_rows_per_unit(int packed_rows);
// Resident CTAs per SM the mma.sync verify kernel is built for (the default grid is this times the SMs).
int mma_ctas_per_sm(int rows_per_unit);
// Dynamic shared memory the mma.sync verify kernel needs.
int mma_smem_bytes(int D, int rows_per_unit, bool kv8 = false);
// keys per work tile of the mma.sync kernel for this unit height (e4m3 caches: 128 for <= 32 rows)
int mma_tile_keys(int rows_per_unit, bool kv8);
cudaError_t launch_verify_mma(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p,
                              int dtype, int grid, cudaStream_t stream);
// The split units' log-sum-exp combine after a verify launched with defer_merge, `grid` = that
// verify's grid; transposed = the tcgen05 kernel's partial layout ([slot][D][128]).
cudaError_t launch_combine_split(const VerifyParams& p, int dtype, int grid, bool transposed, cudaStream_t stream);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);
// Quantising append into an e4m3 cache: code = e4m3(x / scale[h]) (round to nearest even, saturating).
cudaError_t launch_append_e4m3(const AppendArgs& a, const float* k_scale, const float* v_scale, cudaStream_t stream);
// Prefix-tree lookup (insert = false) or insert of B sequences' full blocks.
cudaError_t launch_prefix_cache(bool insert, const int32_t* tokens, const int32_t* seq_starts, const int32_t* block_tables,
                                uint64_t* slot_keys, int32_t* slot_nodes, int64_t capacity, int32_t* node_parent,
                                int32_t* node_depth, int32_t* node_tokens, int32_t* out_blocks, int32_t* out_count,
                                uint32_t* error_word, int B, int bs, int num_blocks, int max_blocks,
                                cudaStream_t stream);
// Lookahead Cache candidate forests and the copy_len update.
cudaError_t launch_lookahead_propose(const int32_t* history, const int32_t* hist_starts, const int32_t* global_tokens,
                                     int64_t global_len, const int32_t* copy_len, int max_match, int B, int C,
                                     int32_t* tokens_out, int32_t* parents_out, int32_t* num_out, uint32_t* error_word,
                                     cudaStream_t stream);
cudaError_t launch_copy_len_update(const int32_t* accept_len, const int32_t* proposed, float* hit, int32_t* copy_len,
                                   int B, int copy_max, float alpha, int batch_ref, cudaStream_t stream);
// Keys per work tile of the tcgen05 verify kernel.
int tc_tile_keys();
// Dynamic shared memory of the tcgen05 verify kernel.
int tc_smem_bytes(int D, bool kv8 = false);
// bf16 query rows -> f16 rows times a power of two per row, and that power's inverse per row (the e4m3
// tcgen05 path's query operand).
cudaError_t launch_q_to_f16(const void* q, void* q16, float* qscale, int64_t rows, int D, cudaStream_t stream);
cudaError_t launch_verify_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const VerifyParams& p, int dtype, int grid, cudaStream_t stream);
// Store the message taco_attn_last_error() returns on this thread.
void set_last_error_message(const char* msg);

}  // namespace taco
