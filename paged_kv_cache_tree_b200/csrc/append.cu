// Paged KV-append: copy each candidate's new K and V rows into its cache slot through the block
// table ("大模型倍速推理引擎 TACO-LLM 的设计与实践", 53ai.com, section "4. 支持 Paged Attention":
// blocks are filled as new tokens are produced). A pure bit copy in 16-byte vectors: one thread per
// 16-byte piece of a (sequence, candidate, KV head) row, so a row of D=128 bf16 is 16 threads
// writing one contiguous 256-byte run of the [NB, Hkv, bs, D] cache.
#include "device_common.cuh"
#include "launchers.h"

namespace taco {

template <int VEC_PER_ROW>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  grid_launch_dependents();  // a verify launched next may start its prologue now
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(a.B) * a.C * a.Hkv * VEC_PER_ROW;
  if (gid >= total) return;
  const int v = static_cast<int>(gid % VEC_PER_ROW);
  const int64_t row = gid / VEC_PER_ROW;          // ((b * C + i) * Hkv + h)
  const int h = static_cast<int>(row % a.Hkv);
  const int64_t bi = row / a.Hkv;                 // b * C + i
  const int b = static_cast<int>(bi / a.C);
  const int s = __ldg(a.slot_offsets + bi);
  if (s < 0) return;
  if (s >= a.max_blocks * a.bs) {
    if (v == 0) atomicOr(a.error_word, TACO_DEVERR_SLOT);
    return;
  }
  const int blk = __ldg(a.block_tables + static_cast<int64_t>(b) * a.max_blocks + s / a.bs);
  if (blk < 0 || blk >= a.num_blocks) {
    if (v == 0) atomicOr(a.error_word, TACO_DEVERR_BLOCK_ID);
    return;
  }
  const int64_t dst = ((static_cast<int64_t>(blk) * a.Hkv + h) * a.bs + s % a.bs) * VEC_PER_ROW + v;
  const uint4 kv = __ldg(static_cast<const uint4*>(a.k_new) + row * VEC_PER_ROW + v);
  const uint4 vv = __ldg(static_cast<const uint4*>(a.v_new) + row * VEC_PER_ROW + v);
  static_cast<uint4*>(a.k_cache)[dst] = kv;
  static_cast<uint4*>(a.v_cache)[dst] = vv;
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const int vec = a.D / 8;
  const int64_t total = static_cast<int64_t>(a.B) * a.C * a.Hkv * vec;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (vec == 16)
    append_kernel<16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  else
    append_kernel<8><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace taco
