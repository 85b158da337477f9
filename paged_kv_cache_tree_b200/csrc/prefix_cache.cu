// Prefix-tree KV lookup for prefill: find the longest run of a prompt's leading full KV blocks that
// earlier requests left in the cache, and insert a finished prefill's blocks.
//
// The pages (618zxw.cn, section "プレフィックスキャッシュ技術を使用してTTFTを削減する"; the 17173xz.com
// overview's prefill paragraph; the tencentcloud.com document's list of techniques) keep earlier
// requests' prefill KV in a prefix tree so that prefill becomes a cache lookup and only the tokens not
// found are computed. Here a node is one full block of bs tokens, identified by the whole token prefix
// it ends, and owns the physical block that holds that prefix's K/V.
//
// Layout (caller-owned device memory):
//   slot_keys  [cap] u64   open addressing with linear probing; 0 = empty
//   slot_nodes [cap] i32   the node (physical block) of a claimed slot, -1 until published
//   node_parent/node_depth [NB] i32, node_tokens [NB, bs] i32, indexed by physical block
// A node's key is a 64-bit hash of its whole token prefix (a polynomial rolling hash whose per-block
// parts are combined by a warp scan, then a 64-bit finaliser). Keys only pick slots: every match is
// confirmed on depth, parent and tokens, so a hash collision never changes a result.
#include "device_common.cuh"
#include "launchers.h"

namespace taco {

namespace {

constexpr uint64_t kHashBase = 0x100000001b3ull;        // odd multiplier of the rolling hash
constexpr uint64_t kDepthSalt = 0x9e3779b97f4a7c15ull;  // mixes the depth into the key
constexpr int kSpinLimit = 1 << 22;                     // bounded wait for a slot's publication

// 64-bit finaliser of MurmurHash3 (its published fmix64 step): every input bit reaches every output bit.
__device__ __forceinline__ uint64_t fmix64(uint64_t x) {
  x ^= x >> 33;
  x *= 0xff51afd7ed558ccdull;
  x ^= x >> 33;
  x *= 0xc4ceb9fe1a85ec53ull;
  x ^= x >> 33;
  return x;
}

__device__ __forceinline__ uint64_t shfl_up_u64(uint64_t v, int off) {
  const uint32_t lo = __shfl_up_sync(0xffffffffu, static_cast<uint32_t>(v), off);
  const uint32_t hi = __shfl_up_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), off);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v), src);
  const uint32_t hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Per-block hashes of full blocks c0 + lane (lane < count) of one sequence and their inclusive scan
// with a zero carry. Prefix hash of blocks 0..j: H_j = H_(j-1) * base^bs + h_j, h_j the block's own
// polynomial hash; the recurrence is a scan with (a, q) o (b, r) = (a * r + b, q * r). On return a
// lane holds a = H of blocks c0..j alone and q = base^(bs * (j - c0 + 1)); H_j = carry * q + a.
__device__ __forceinline__ void chunk_scan(const int32_t* seq, int c0, int count, int bs, uint64_t base_bs, int lane,
                                           uint64_t& a, uint64_t& q) {
  a = 0;
  q = 1;
  if (lane < count) {
    const int32_t* t = seq + static_cast<int64_t>(c0 + lane) * bs;
    for (int i = 0; i < bs; ++i) a = a * kHashBase + (static_cast<uint64_t>(static_cast<uint32_t>(__ldg(t + i))) + 1ull);
    q = base_bs;
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint64_t a2 = shfl_up_u64(a, off);
    const uint64_t q2 = shfl_up_u64(q, off);
    if (lane >= off) {
      a = a2 * q + a;
      q = q2 * q;
    }
  }
}

__device__ __forceinline__ uint64_t block_key(uint64_t H, int j) {
  return fmix64(H + static_cast<uint64_t>(j + 1) * kDepthSalt) | 1ull;
}

// Keys of full blocks c0 + lane (lane < count) given the prefix hash `carry` of the blocks before c0;
// updates carry to H of the chunk's last block. Lanes past count get 0.
__device__ __forceinline__ uint64_t chunk_keys(const int32_t* seq, int c0, int count, int bs, uint64_t base_bs,
                                               uint64_t& carry, int lane) {
  uint64_t a, q;
  chunk_scan(seq, c0, count, bs, base_bs, lane, a, q);
  const uint64_t H = carry * q + a;
  carry = shfl_u64(H, count - 1);
  return lane < count ? block_key(H, c0 + lane) : 0ull;
}

// Token-by-token equality of a block, loads issued eight at a time (one dependent round trip per
// eight tokens rather than per token).
__device__ __forceinline__ bool block_tokens_equal(const int32_t* a, const int32_t* node_tok, int bs) {
  int i = 0;
  for (; i + 8 <= bs; i += 8) {
    int32_t x[8], y[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x[k] = __ldg(a + i + k);
      y[k] = __ldg(node_tok + i + k);
    }
    bool eq = true;
#pragma unroll
    for (int k = 0; k < 8; ++k) eq &= x[k] == y[k];
    if (!eq) return false;
  }
  bool eq = true;
  for (; i < bs; ++i) eq &= __ldg(a + i) == __ldg(node_tok + i);
  return eq;
}

struct PrefixArgs {
  const int32_t* tokens;
  const int32_t* seq_starts;
  const int32_t* block_tables;
  uint64_t* slot_keys;
  int32_t* slot_nodes;
  int32_t* node_parent;
  int32_t* node_depth;
  int32_t* node_tokens;
  int32_t* out_blocks;
  int32_t* out_matched;
  uint32_t* error_word;
  int64_t cap;
  int B, bs, num_blocks, max_blocks;
};

__device__ __forceinline__ int full_blocks(const PrefixArgs& a, int b, int lane, int64_t& s0) {
  s0 = __ldg(a.seq_starts + b);
  const int64_t n = static_cast<int64_t>(__ldg(a.seq_starts + b + 1)) - s0;
  if (n < 0 || s0 < 0) {
    if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_CONTEXT_LEN);
    return 0;
  }
  const int64_t nf = n / a.bs;
  return static_cast<int>(nf < a.max_blocks ? nf : a.max_blocks);
}

__device__ __forceinline__ uint64_t base_pow_bs(int bs) {
  uint64_t r = 1;
  for (int i = 0; i < bs; ++i) r *= kHashBase;
  return r;
}

// --------------------------------------------------------------------------------------------- lookup
constexpr int kLookupWarps = 8;

// Slot of the node for block j with key `key`, depth j, the given tokens and (if want_parent > -2) the
// given parent: the first such node on the key's probe chain, or -1. `second` reports whether another
// node with equal key, depth and tokens follows it on the chain (only when want_parent == -2).
__device__ __forceinline__ int probe_node(const PrefixArgs& a, uint64_t key, int j, const int32_t* tok, int want_parent,
                                          bool& second) {
  const uint64_t mask = static_cast<uint64_t>(a.cap) - 1;
  uint64_t slot = key & mask;
  int node = -1;
  second = false;
  for (int64_t it = 0; it < a.cap; ++it) {
    const uint64_t k = __ldg(a.slot_keys + slot);
    if (k == 0ull) break;
    if (k == key) {
      const int nd = __ldg(a.slot_nodes + slot);
      if (nd >= 0 && nd < a.num_blocks && __ldg(a.node_depth + nd) == j &&
          (want_parent == -2 || __ldg(a.node_parent + nd) == want_parent) &&
          block_tokens_equal(tok, a.node_tokens + static_cast<int64_t>(nd) * a.bs, a.bs)) {
        if (node < 0) {
          node = nd;
          if (want_parent != -2) break;
        } else {
          second = true;
          break;
        }
      }
    }
    slot = (slot + 1) & mask;
  }
  return node;
}

// One CTA of 8 warps per prompt, 256 blocks per round: each warp hashes and scans a chunk of 32 blocks,
// the chunks' carries combine through shared memory, every block probes its chain in parallel, and
// the parent links then decide the matched run (the first block whose node is missing or hangs from
// another parent ends it). A block with two candidates (a full 64-bit collision of two prefixes ending
// in the same tokens) is resolved in order by warp 0 with its known parent.
__global__ void __launch_bounds__(kLookupWarps * 32) prefix_lookup_kernel(PrefixArgs a) {
  constexpr int RB = kLookupWarps * 32;
  __shared__ uint64_t sh_A[kLookupWarps], sh_Q[kLookupWarps];
  __shared__ uint64_t sh_key[RB];
  __shared__ int sh_node[RB];
  __shared__ unsigned char sh_multi[RB];
  __shared__ int sh_any_multi, sh_first_bad;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t s0;
  const int nfull = full_blocks(a, b, threadIdx.x, s0);
  const int32_t* seq = a.tokens + s0;
  const uint64_t base_bs = base_pow_bs(a.bs);
  int32_t* out = a.out_blocks + static_cast<int64_t>(b) * a.max_blocks;
  uint64_t carry = 0;
  int prev_node = -1;
  int matched = nfull;
  for (int r0 = 0; r0 < nfull; r0 += RB) {
    const int rcount = nfull - r0 < RB ? nfull - r0 : RB;
    int count = rcount - warp * 32;
    count = count < 0 ? 0 : (count > 32 ? 32 : count);
    const int c0 = r0 + warp * 32;
    uint64_t av, qv;
    chunk_scan(seq, c0, count, a.bs, base_bs, lane, av, qv);
    // the chunk's own hash and multiplier (a zero-length chunk gives 0 and 1)
    const uint64_t chunk_a = shfl_u64(av, count > 0 ? count - 1 : 0);
    const uint64_t chunk_q = shfl_u64(qv, count > 0 ? count - 1 : 0);
    if (lane == 0) {
      sh_A[warp] = chunk_a;
      sh_Q[warp] = chunk_q;
    }
    if (threadIdx.x == 0) {
      sh_any_multi = 0;
      sh_first_bad = rcount;
    }
    __syncthreads();
    uint64_t cw = carry, next_carry = carry;
#pragma unroll
    for (int i = 0; i < kLookupWarps; ++i) {
      if (i < warp) cw = cw * sh_Q[i] + sh_A[i];
      next_carry = next_carry * sh_Q[i] + sh_A[i];
    }
    const int idx = warp * 32 + lane;
    const int j = c0 + lane;
    const bool active = lane < count;
    const uint64_t key = active ? block_key(cw * qv + av, j) : 0ull;
    int node = -1;
    bool multi = false;
    if (active) node = probe_node(a, key, j, seq + static_cast<int64_t>(j) * a.bs, -2, multi);
    sh_key[idx] = key;
    sh_node[idx] = node;
    sh_multi[idx] = multi ? 1 : 0;
    if (multi) atomicOr(&sh_any_multi, 1);
    __syncthreads();
    if (sh_any_multi) {
      if (warp == 0) {
        for (int x = 0; x < rcount; ++x) {
          if (sh_multi[x]) {
            if (lane == 0) {
              bool unused;
              const int want = x == 0 ? prev_node : sh_node[x - 1];
              sh_node[x] = probe_node(a, sh_key[x], r0 + x, seq + static_cast<int64_t>(r0 + x) * a.bs, want, unused);
            }
            __syncwarp();
          }
        }
      }
      __syncthreads();
    }
    if (active) {
      const int nd = sh_node[idx];
      const int expect = idx == 0 ? prev_node : sh_node[idx - 1];
      if (!(nd >= 0 && __ldg(a.node_parent + nd) == expect)) atomicMin(&sh_first_bad, idx);
    }
    __syncthreads();
    const int fb = sh_first_bad;
    if (active && idx < fb) out[j] = sh_node[idx];
    if (fb < rcount) {
      matched = r0 + fb;
      break;
    }
    prev_node = sh_node[rcount - 1];
    carry = next_carry;
    __syncthreads();
  }
  for (int jj = matched + static_cast<int>(threadIdx.x); jj < a.max_blocks; jj += blockDim.x) out[jj] = -1;
  if (threadIdx.x == 0) a.out_matched[b] = matched;
}

// --------------------------------------------------------------------------------------------- insert
// One warp per sequence, its full blocks in order. Probing a block's chain: an empty slot is claimed
// with a compare-and-swap and the sequence's own block becomes the node (data written, then the slot
// published); a slot with the same key is waited for until published (bounded) and reused when depth,
// parent and tokens match. Every other slot is skipped.
__global__ void __launch_bounds__(256) prefix_insert_kernel(PrefixArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.B) return;
  const int b = warp;
  int64_t s0;
  const int nfull = full_blocks(a, b, lane, s0);
  const int32_t* seq = a.tokens + s0;
  const uint64_t base_bs = base_pow_bs(a.bs);
  const uint64_t mask = static_cast<uint64_t>(a.cap) - 1;
  const int32_t* table = a.block_tables + static_cast<int64_t>(b) * a.max_blocks;
  int32_t* out = a.out_blocks + static_cast<int64_t>(b) * a.max_blocks;
  uint64_t carry = 0;
  int parent = -1;
  int done = 0;
  bool stop = false;
  uint64_t key_lane = 0;
  for (int j = 0; j < nfull && !stop; ++j) {
    if ((j & 31) == 0) {
      const int count = nfull - j < 32 ? nfull - j : 32;
      key_lane = chunk_keys(seq, j, count, a.bs, base_bs, carry, lane);
    }
    const uint64_t key = shfl_u64(key_lane, j & 31);
    const int own = __ldg(table + j);
    if (own < 0 || own >= a.num_blocks) {
      if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_BLOCK_ID);
      break;
    }
    const int32_t* tok = seq + static_cast<int64_t>(j) * a.bs;
    uint64_t slot = key & mask;
    int found = -1;
    for (int64_t it = 0; it < a.cap && found < 0 && !stop; ++it) {
      uint64_t k = 0;
      // one compare-and-swap both reads the slot and, when it is empty, claims it (0 comes back)
      if (lane == 0) k = atomicCAS(reinterpret_cast<unsigned long long*>(a.slot_keys + slot), 0ull, key);
      k = shfl_u64(k, 0);
      if (k == 0ull) {
        // claimed: write the node, then publish it
        for (int i = lane; i < a.bs; i += 32) a.node_tokens[static_cast<int64_t>(own) * a.bs + i] = __ldg(tok + i);
        if (lane == 0) {
          a.node_parent[own] = parent;
          a.node_depth[own] = j;
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicExch(a.slot_nodes + slot, own);
        found = own;
        break;
      }
      if (k == key) {
        int nd = -1;
        if (lane == 0) {
          for (int spin = 0; spin < kSpinLimit; ++spin) {
            nd = atomicAdd(a.slot_nodes + slot, 0);
            if (nd >= 0) break;
            __nanosleep(32);
          }
        }
        nd = __shfl_sync(0xffffffffu, nd, 0);
        if (nd < 0) {
          if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_WAIT_TIMEOUT);
          stop = true;
          break;
        }
        __threadfence();
        bool same = nd < a.num_blocks && __ldcg(a.node_depth + nd) == j && __ldcg(a.node_parent + nd) == parent;
        if (same) {
          bool eq = true;
          for (int i = lane; i < a.bs; i += 32) eq &= (__ldg(tok + i) == __ldcg(a.node_tokens + static_cast<int64_t>(nd) * a.bs + i));
          same = __all_sync(0xffffffffu, eq);
        }
        if (same) {
          found = nd;
          break;
        }
      }
      slot = (slot + 1) & mask;
    }
    if (stop) break;
    if (found < 0) {
      if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_TABLE_FULL);
      break;
    }
    if (lane == 0) out[j] = found;
    parent = found;
    done = j + 1;
  }
  for (int jj = done + lane; jj < a.max_blocks; jj += 32) out[jj] = -1;
  if (a.out_matched != nullptr && lane == 0) a.out_matched[b] = done;
}

}  // namespace

cudaError_t launch_prefix_cache(bool insert, const int32_t* tokens, const int32_t* seq_starts, const int32_t* block_tables,
                                uint64_t* slot_keys, int32_t* slot_nodes, int64_t capacity, int32_t* node_parent,
                                int32_t* node_depth, int32_t* node_tokens, int32_t* out_blocks, int32_t* out_count,
                                uint32_t* error_word, int B, int bs, int num_blocks, int max_blocks,
                                cudaStream_t stream) {
  PrefixArgs a{tokens, seq_starts, block_tables, slot_keys, slot_nodes, node_parent, node_depth, node_tokens,
               out_blocks, out_count, error_word, capacity, B, bs, num_blocks, max_blocks};
  if (insert)
    prefix_insert_kernel<<<(B * 32 + 255) / 256, 256, 0, stream>>>(a);
  else
    prefix_lookup_kernel<<<B, kLookupWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace taco
