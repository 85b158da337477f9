// The step after the verify: tree masks from parent arrays, the target's argmax over the vocabulary,
// and greedy acceptance of the longest correct root-to-node path of each candidate tree with the
// slot offsets that compact the accepted candidates' K/V into the contiguous tail of the cache.
//
// The pages ("大模型倍速推理引擎 TACO-LLM 的设计与实践", sections "TACO-LLM 如何解决大模型推理瓶颈?",
// "优化方案设计思路" and "优化策略总结") have the target model validate candidate tokens obtained
// ahead of time, organised as a forest, and measure the candidates' hit length. The acceptance rule
// is the plain greedy one: candidate i is correct iff its token is the target's argmax after its
// parent (after the prefix for a root); a candidate is accepted iff it and all its ancestors are
// correct; the hit is the deepest accepted candidate (smallest index on ties); the target's argmax
// after the hit (after the prefix when nothing is accepted) is the bonus token.
#include <float.h>

#include "device_common.cuh"
#include "launchers.h"

namespace taco {

// ---------------------------------------------------------------------------------------------- masks
// One warp per sequence, lane i = candidate i: the word of i has bit j set iff j is i or one of its
// ancestors. A parent outside [-1, i) is reported and ends the walk.
__global__ void __launch_bounds__(256) tree_mask_kernel(MaskArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.B) return;
  const int b = warp;
  int n = __ldg(a.num_candidates + b);
  if (n < 0 || n > a.C) {
    if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_NUM_CAND);
    n = n < 0 ? 0 : a.C;
  }
  if (lane >= a.C) return;
  const int32_t* par = a.parents + static_cast<int64_t>(b) * a.C;
  uint32_t word = 0;
  if (lane < n) {
    int j = lane;
    for (int step = 0; step < 32 && j >= 0; ++step) {
      word |= 1u << j;
      const int pj = __ldg(par + j);
      if (pj < -1 || pj >= j) {
        atomicOr(a.error_word, TACO_DEVERR_PARENT);
        break;
      }
      j = pj;
    }
  }
  a.mask_out[static_cast<int64_t>(b) * a.C + lane] = word;
}

// ---------------------------------------------------------------------------------------------- argmax
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) {
  return __half2float(x);
}

// (value, index) with the larger value winning and, on equal values, the smaller index. NaN never
// wins (it compares false); an index of INT_MAX means "no number seen".
__device__ __forceinline__ void arg_better(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

constexpr int kArgmaxThreads = 1024;
constexpr int kArgmaxUnroll = 8;

// One CTA per row. VEC: 8 elements per 16-byte load (row starts 16-byte aligned) or 1 (any layout).
template <typename T, int VEC>
__global__ void __launch_bounds__(kArgmaxThreads) argmax_kernel(const T* __restrict__ logits, int64_t rows, int vocab,
                                                                int32_t* __restrict__ out) {
  __shared__ float sv[32];
  __shared__ int si[32];
  const int64_t row = blockIdx.x;
  if (row >= rows) return;
  const T* x = logits + row * static_cast<int64_t>(vocab);
  float best = -INFINITY;
  int bi = INT_MAX;
  const int tid = threadIdx.x;
  if (VEC == 8) {
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const int nvec = vocab / 8;
    // each thread walks its vectors in increasing order, so a strict > keeps its first maximum
    for (int v0 = tid; v0 < nvec; v0 += kArgmaxThreads * kArgmaxUnroll) {
      uint4 buf[kArgmaxUnroll];
#pragma unroll
      for (int u = 0; u < kArgmaxUnroll; ++u) {
        const int v = v0 + u * kArgmaxThreads;
        buf[u] = v < nvec ? __ldcs(xv + v) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
      }
#pragma unroll
      for (int u = 0; u < kArgmaxUnroll; ++u) {
        const int v = v0 + u * kArgmaxThreads;
        if (v >= nvec) break;
        const T* e = reinterpret_cast<const T*>(&buf[u]);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float f = to_f32<T>(e[k]);
          if (f > best) {
            best = f;
            bi = v * 8 + k;
          }
        }
      }
    }
  } else {
    for (int k = tid; k < vocab; k += kArgmaxThreads) {
      const float f = to_f32<T>(x[k]);
      if (f > best) {
        best = f;
        bi = k;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, best, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
    arg_better(best, bi, v2, i2);
  }
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
    sv[warp] = best;
    si[warp] = bi;
  }
  __syncthreads();
  if (warp == 0) {
    best = lane < kArgmaxThreads / 32 ? sv[lane] : -INFINITY;
    bi = lane < kArgmaxThreads / 32 ? si[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, best, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
      arg_better(best, bi, v2, i2);
    }
    if (lane == 0) out[row] = bi == INT_MAX ? 0 : bi;
  }
}

// ---------------------------------------------------------------------------------------------- accept
// One warp per sequence, lane i = candidate i (C <= 32). Accepted flags, depths and ancestor masks
// follow parent links; a parent always has a smaller index, so 32 rounds of shuffles settle them.
__global__ void __launch_bounds__(256) accept_kernel(AcceptArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.B) return;
  const int b = warp;
  const int C = a.C;
  int n = __ldg(a.num_candidates + b);
  const int L = __ldg(a.context_lens + b);
  if (n < 0 || n > C || n > L) {
    if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_NUM_CAND);
    n = n < 0 ? 0 : (n > C ? C : n);
    if (n > L) n = L < 0 ? 0 : L;
  }
  const int64_t base = static_cast<int64_t>(b) * C;
  const int32_t* amax = a.target_argmax + static_cast<int64_t>(b) * (C + 1);
  const bool live = lane < n;
  int par = live ? __ldg(a.parents + base + lane) : -1;
  bool ok_parent = true;
  if (live && (par < -1 || par >= lane)) {
    atomicOr(a.error_word, TACO_DEVERR_PARENT);
    ok_parent = false;
    par = -1;
  }
  const bool correct = live && ok_parent && __ldg(a.tokens + base + lane) == __ldg(amax + (par < 0 ? 0 : par + 1));
  bool acc = correct;
  int depth = 1;
  uint32_t anc = 1u << lane;
#pragma unroll 1
  for (int it = 0; it < 32; ++it) {
    const int src = par < 0 ? lane : par;
    const bool pacc = __shfl_sync(0xffffffffu, acc, src);
    const int pdepth = __shfl_sync(0xffffffffu, depth, src);
    const uint32_t panc = __shfl_sync(0xffffffffu, anc, src);
    if (par >= 0) {
      acc = correct && pacc;
      depth = pdepth + 1;
      anc = (1u << lane) | panc;
    }
  }
  // deepest accepted candidate, smallest index on ties
  const uint32_t key = acc ? (static_cast<uint32_t>(depth) << 8) | static_cast<uint32_t>(31 - lane) : 0u;
  const uint32_t top = __reduce_max_sync(0xffffffffu, key);
  const int best = top ? 31 - static_cast<int>(top & 0xffu) : -1;
  const int accept_len = top ? static_cast<int>(top >> 8) : 0;
  const uint32_t best_anc = __shfl_sync(0xffffffffu, anc, best < 0 ? 0 : best);
  const bool on_path = best >= 0 && live && ((best_anc >> lane) & 1u);
  const int P = L - n;
  if (lane < C) {
    a.slot_offsets_out[base + lane] = on_path ? P + depth - 1 : -1;
    if (lane >= accept_len) a.accepted_path[base + lane] = -1;
  }
  if (on_path) a.accepted_path[base + depth - 1] = lane;
  if (lane == 0) {
    a.accept_len[b] = accept_len;
    a.bonus_token[b] = __ldg(amax + (best < 0 ? 0 : best + 1));
  }
}

// ---------------------------------------------------------------------------------------------- launchers
cudaError_t launch_tree_masks(const MaskArgs& a, cudaStream_t stream) {
  const int blocks = (a.B * 32 + 255) / 256;
  tree_mask_kernel<<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_argmax(const void* logits, int dtype, int64_t rows, int vocab, int32_t* out, cudaStream_t stream) {
  const bool vec = (reinterpret_cast<uintptr_t>(logits) % 16 == 0) && (vocab % 8 == 0);
  const dim3 grid(static_cast<unsigned>(rows));
  if (dtype == TACO_DTYPE_BF16) {
    const auto* x = static_cast<const __nv_bfloat16*>(logits);
    if (vec)
      argmax_kernel<__nv_bfloat16, 8><<<grid, kArgmaxThreads, 0, stream>>>(x, rows, vocab, out);
    else
      argmax_kernel<__nv_bfloat16, 1><<<grid, kArgmaxThreads, 0, stream>>>(x, rows, vocab, out);
  } else {
    const auto* x = static_cast<const __half*>(logits);
    if (vec)
      argmax_kernel<__half, 8><<<grid, kArgmaxThreads, 0, stream>>>(x, rows, vocab, out);
    else
      argmax_kernel<__half, 1><<<grid, kArgmaxThreads, 0, stream>>>(x, rows, vocab, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_accept(const AcceptArgs& a, cudaStream_t stream) {
  const int blocks = (a.B * 32 + 255) / 256;
  accept_kernel<<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace taco
