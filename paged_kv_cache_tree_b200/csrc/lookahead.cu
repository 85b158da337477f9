// Batched Lookahead Cache: candidate forests for the verify, from earlier occurrences of each
// sequence's most recent tokens in its own history (local cache) and in a shared token array (global
// cache), and the per-sequence copy_len update after each verify.
//
// The pages (53ai.com workshop page, "整体方案分为两大部分", item 1 "基于批处理的 Lookahead Cache" and
// the paragraphs after it) predict a whole batch at once from local and global caches queried by match
// length, copy a preset number of tokens that is penalised adaptively from batch size and hit rate, and
// propose a forest. Definitions used here:
//  - match: the longest m <= max_match such that the last m tokens of the history occur in the cache
//    ending at a position e that has a following token (local: e < n, an earlier occurrence);
//    tokens below 0 (separators) never match;
//  - occurrences of that m are taken most recent first, each contributing the following tokens (at most
//    copy_len, stopping before a separator or the end) as a path;
//  - local paths, then global ones, are merged into a trie of at most C nodes numbered in creation order.
#include "device_common.cuh"
#include "launchers.h"

namespace taco {

namespace {

constexpr int kLaThreads = 256;
constexpr int kLaMaxKey = 16;
constexpr int kLaMaxOcc = 1024;   // occurrences gathered and sorted in shared memory per cache

struct LaArgs {
  const int32_t* history;
  const int32_t* hist_starts;
  const int32_t* global_tokens;
  int64_t global_len;
  const int32_t* copy_len;
  int32_t* tokens_out;
  int32_t* parents_out;
  int32_t* num_out;
  uint32_t* error_word;
  int B, C, max_match;
};

// Length of the common run of src[.. e) and the key's last tokens (key[mk - 1] is the latest), capped at
// mk and at e; 0 when src[e] (the following token) is a separator.
__device__ __forceinline__ int match_len(const int32_t* src, int64_t e, const int32_t* key, int mk) {
  if (__ldg(src + e) < 0) return 0;
  const int kmax = static_cast<int64_t>(mk) < e ? mk : static_cast<int>(e);
  int ml = 0;
  for (int k = 1; k <= kmax; ++k) {
    const int32_t t = __ldg(src + e - k);
    if (t < 0 || t != key[mk - k]) break;
    ml = k;
  }
  return ml;
}

// Calls f(e, ml) for every end position e in [1, len) strided over the CTA whose match length ml is
// at least 1, four positions per thread at a time so that their first loads overlap (most positions
// fail on the last key token).
template <typename F>
__device__ __forceinline__ void for_each_match(const int32_t* src, int64_t len, const int32_t* key, int mk, int tid,
                                               F f) {
  const int32_t last = key[mk - 1];
  for (int64_t e0 = 1 + tid; e0 < len; e0 += 4 * kLaThreads) {
    int32_t nx[4], lt[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = e0 + static_cast<int64_t>(u) * kLaThreads;
      nx[u] = e < len ? __ldg(src + e) : -1;
      lt[u] = e < len ? __ldg(src + e - 1) : -1;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (nx[u] >= 0 && lt[u] == last && lt[u] >= 0) {
        const int64_t e = e0 + static_cast<int64_t>(u) * kLaThreads;
        f(e, match_len(src, e, key, mk));
      }
    }
  }
}

// Warp 0's trie: lane i holds node i (parent, token) for i < count. Inserts the path src[e ..) of at
// most copy_len tokens; returns false once the trie is full (C nodes and a token with no node).
__device__ __forceinline__ bool insert_path(const int32_t* src, int64_t len, int64_t e, int copy_len, int C, int lane,
                                            int& count, int& my_par, int& my_tok) {
  int parent = -1;
  for (int s = 0; s < copy_len && e + s < len; ++s) {
    const int32_t t = __ldg(src + e + s);
    if (t < 0) break;
    const uint32_t hit = __ballot_sync(0xffffffffu, lane < count && my_par == parent && my_tok == t);
    if (hit) {
      parent = __ffs(hit) - 1;
      continue;
    }
    if (count >= C) return false;
    if (lane == count) {
      my_par = parent;
      my_tok = t;
    }
    parent = count;
    ++count;
  }
  return true;
}

__global__ void __launch_bounds__(kLaThreads) lookahead_propose_kernel(LaArgs a) {
  __shared__ int32_t sh_key[kLaMaxKey];
  __shared__ int32_t sh_occ[kLaMaxOcc];
  __shared__ int sh_best, sh_count, sh_full, sh_chunk;
  __shared__ int sh_warp_cnt[kLaThreads / 32];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t s0 = __ldg(a.hist_starts + b);
  int64_t n = static_cast<int64_t>(__ldg(a.hist_starts + b + 1)) - s0;
  if (n < 0 || s0 < 0) {
    if (tid == 0) atomicOr(a.error_word, TACO_DEVERR_CONTEXT_LEN);
    n = 0;
  }
  const int32_t* hist = a.history + (s0 < 0 ? 0 : s0);
  const int mk = static_cast<int>(n < a.max_match ? n : a.max_match);
  if (tid < mk) sh_key[tid] = __ldg(hist + n - mk + tid);
  if (tid == 0) sh_full = 0;
  const int copy = __ldg(a.copy_len + b);
  int count = 0, my_par = -1, my_tok = -1;   // warp 0's trie
  __syncthreads();

  for (int which = 0; which < 2 && mk > 0 && copy > 0; ++which) {
    const int32_t* src = which == 0 ? hist : a.global_tokens;
    const int64_t len = which == 0 ? n : a.global_len;
    if (len < 2 || src == nullptr) continue;
    // longest match over every end position with a following token
    if (tid == 0) sh_best = 0;
    __syncthreads();
    int best = 0;
    for_each_match(src, len, sh_key, mk, tid, [&](int64_t, int ml) { best = ml > best ? ml : best; });
    if (best > 0) atomicMax(&sh_best, best);
    __syncthreads();
    const int m = sh_best;
    if (m == 0) continue;
    // gather the occurrences of length m
    if (tid == 0) sh_count = 0;
    __syncthreads();
    for_each_match(src, len, sh_key, mk, tid, [&](int64_t e, int ml) {
      if (ml >= m) {
        const int idx = atomicAdd(&sh_count, 1);
        if (idx < kLaMaxOcc) sh_occ[idx] = static_cast<int32_t>(e);
      }
    });
    __syncthreads();
    const int cnt = sh_count;
    if (cnt <= kLaMaxOcc) {
      // bitonic sort, descending, padded with -1 to a power of two
      int P2 = 1;
      while (P2 < cnt) P2 <<= 1;
      for (int i = cnt + tid; i < P2; i += kLaThreads) sh_occ[i] = -1;
      __syncthreads();
      for (int k = 2; k <= P2; k <<= 1) {
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
          for (int i = tid; i < P2; i += kLaThreads) {
            const int l = i ^ jj;
            if (l > i) {
              const bool desc = (i & k) == 0;
              const int32_t x = sh_occ[i], y = sh_occ[l];
              if (desc ? (x < y) : (x > y)) {
                sh_occ[i] = y;
                sh_occ[l] = x;
              }
            }
          }
          __syncthreads();
        }
      }
      if (warp == 0) {
        bool room = sh_full == 0;
        for (int i = 0; i < cnt && room; ++i) room = insert_path(src, len, sh_occ[i], copy, a.C, lane, count, my_par, my_tok);
        if (lane == 0 && !room) sh_full = 1;
      }
      __syncthreads();
    } else {
      // too many to sort here: walk the positions downwards a chunk at a time, in order
      for (int64_t base = len - 1; base >= 1; base -= kLaThreads) {
        if (sh_full) break;
        const int64_t e = base - tid;
        const bool occ = e >= 1 && match_len(src, e, sh_key, mk) >= m;
        const uint32_t bal = __ballot_sync(0xffffffffu, occ);
        if (lane == 0) sh_warp_cnt[warp] = __popc(bal);
        __syncthreads();
        int off = 0;
        for (int w = 0; w < warp; ++w) off += sh_warp_cnt[w];
        if (occ) sh_occ[off + __popc(bal & ((1u << lane) - 1u))] = static_cast<int32_t>(e);
        if (tid == kLaThreads - 1) sh_chunk = off + __popc(bal);
        __syncthreads();
        if (warp == 0) {
          bool room = true;
          const int cc = sh_chunk;
          for (int i = 0; i < cc && room; ++i) room = insert_path(src, len, sh_occ[i], copy, a.C, lane, count, my_par, my_tok);
          if (lane == 0 && !room) sh_full = 1;
        }
        __syncthreads();
      }
    }
    if (sh_full) break;
  }
  if (warp == 0) {
    const int64_t row = static_cast<int64_t>(b) * a.C;
    if (lane < a.C) {
      a.tokens_out[row + lane] = lane < count ? my_tok : -1;
      a.parents_out[row + lane] = lane < count ? my_par : -1;
    }
    if (lane == 0) a.num_out[b] = count;
  }
}

// hit <- (1 - alpha) hit + alpha * accepted / max(1, proposed);
// copy_len = clamp(floor(copy_max * hit * min(1, batch_ref / B) + 0.5), 1, copy_max), each step rounded
// to float32 (no fused multiply-add), so that the integer matches any float32 evaluation in this order.
__global__ void copy_len_kernel(const int32_t* accept_len, const int32_t* proposed, float* hit, int32_t* copy_len, int B,
                                int copy_max, float alpha, int batch_ref) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const float acc = static_cast<float>(accept_len[b]);
  const float prop = fmaxf(static_cast<float>(proposed[b]), 1.f);
  const float rate = __fdiv_rn(acc, prop);
  const float h = __fadd_rn(__fmul_rn(__fadd_rn(1.f, -alpha), hit[b]), __fmul_rn(alpha, rate));
  hit[b] = h;
  const float scale = fminf(1.f, __fdiv_rn(static_cast<float>(batch_ref), static_cast<float>(B)));
  const float x = __fadd_rn(__fmul_rn(__fmul_rn(static_cast<float>(copy_max), h), scale), 0.5f);
  int c = static_cast<int>(floorf(x));
  c = c < 1 ? 1 : (c > copy_max ? copy_max : c);
  copy_len[b] = c;
}

}  // namespace

cudaError_t launch_lookahead_propose(const int32_t* history, const int32_t* hist_starts, const int32_t* global_tokens,
                                     int64_t global_len, const int32_t* copy_len, int max_match, int B, int C,
                                     int32_t* tokens_out, int32_t* parents_out, int32_t* num_out, uint32_t* error_word,
                                     cudaStream_t stream) {
  LaArgs a{history, hist_starts, global_tokens, global_len, copy_len, tokens_out, parents_out, num_out, error_word,
           B, C, max_match};
  lookahead_propose_kernel<<<B, kLaThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_copy_len_update(const int32_t* accept_len, const int32_t* proposed, float* hit, int32_t* copy_len,
                                   int B, int copy_max, float alpha, int batch_ref, cudaStream_t stream) {
  copy_len_kernel<<<(B + 255) / 256, 256, 0, stream>>>(accept_len, proposed, hit, copy_len, B, copy_max, alpha,
                                                       batch_ref);
  return cudaGetLastError();
}

}  // namespace taco
