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
  int s;
  if (a.slot_offsets != nullptr) {
    s = __ldg(a.slot_offsets + bi);
  } else {
    const int i = static_cast<int>(bi % a.C);
    const int n = __ldg(a.num_candidates + b), L = __ldg(a.context_lens + b);
    s = (i < n && n <= a.C && n <= L) ? L - n + i : -1;  // slots [L - n, L) with n <= C
  }
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

// Quantising append into an e4m3 cache [NB, Hkv, bs, D] (one byte per value): one thread per 16-byte
// piece (8 values) of a (sequence, candidate, KV head) row of k_new / v_new, writing 8 bytes; each
// value is divided by its KV head's scale (float32, correctly rounded) and rounded to e4m3.
template <typename T, int VEC_PER_ROW>
__global__ void __launch_bounds__(256) append_e4m3_kernel(AppendArgs a, const float* k_scale, const float* v_scale) {
  grid_launch_dependents();
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(a.B) * a.C * a.Hkv * VEC_PER_ROW;
  if (gid >= total) return;
  const int v = static_cast<int>(gid % VEC_PER_ROW);
  const int64_t row = gid / VEC_PER_ROW;          // ((b * C + i) * Hkv + h)
  const int h = static_cast<int>(row % a.Hkv);
  const int64_t bi = row / a.Hkv;
  const int b = static_cast<int>(bi / a.C);
  int s;
  if (a.slot_offsets != nullptr) {
    s = __ldg(a.slot_offsets + bi);
  } else {
    const int i = static_cast<int>(bi % a.C);
    const int n = __ldg(a.num_candidates + b), L = __ldg(a.context_lens + b);
    s = (i < n && n <= a.C && n <= L) ? L - n + i : -1;  // slots [L - n, L) with n <= C
  }
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
  const float ks = __ldg(k_scale + h), vs = __ldg(v_scale + h);
  const uint4 kin = __ldg(static_cast<const uint4*>(a.k_new) + row * VEC_PER_ROW + v);
  const uint4 vin = __ldg(static_cast<const uint4*>(a.v_new) + row * VEC_PER_ROW + v);
  // 8 bytes per thread: cache row (blk, h, slot) is D bytes, this piece starts at byte v * 8
  const int64_t dst = ((static_cast<int64_t>(blk) * a.Hkv + h) * a.bs + s % a.bs) * VEC_PER_ROW + v;
  static_cast<uint2*>(a.k_cache)[dst] = quantise_e4m3x8<T>(kin, ks);
  static_cast<uint2*>(a.v_cache)[dst] = quantise_e4m3x8<T>(vin, vs);
}

cudaError_t launch_append_e4m3(const AppendArgs& a, const float* k_scale, const float* v_scale, cudaStream_t stream) {
  const int vec = a.D / 8;
  const int64_t total = static_cast<int64_t>(a.B) * a.C * a.Hkv * vec;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  const bool bf16 = a.dtype == TACO_DTYPE_BF16;
  if (vec == 16) {
    if (bf16)
      append_e4m3_kernel<__nv_bfloat16, 16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a, k_scale, v_scale);
    else
      append_e4m3_kernel<__half, 16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a, k_scale, v_scale);
  } else {
    if (bf16)
      append_e4m3_kernel<__nv_bfloat16, 8><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a, k_scale, v_scale);
    else
      append_e4m3_kernel<__half, 8><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a, k_scale, v_scale);
  }
  return cudaGetLastError();
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
