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
};

// Rows of packed queries one unit of the mma.sync verify kernel covers for a given G * C.
int mma_rows_per_unit(int packed_rows);
// Dynamic shared memory the mma.sync verify kernel needs.
int mma_smem_bytes(int D, int rows_per_unit);
cudaError_t launch_verify_mma(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p,
                              int dtype, int grid, cudaStream_t stream);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);
// Keys per work tile of the tcgen05 verify kernel.
int tc_tile_keys();
// Dynamic shared memory of the tcgen05 verify kernel.
int tc_smem_bytes(int D);
cudaError_t launch_verify_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const VerifyParams& p, int dtype, int grid, cudaStream_t stream);
// Store the message taco_attn_last_error() returns on this thread.
void set_last_error_message(const char* msg);

}  // namespace taco
