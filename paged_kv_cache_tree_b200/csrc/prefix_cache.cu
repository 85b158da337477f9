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
    // the block's tokens are loaded eight at a time before they are hashed, so that a block costs one
    // dependent round trip per eight tokens rather than per token
    const int32_t* t = seq + static_cast<int64_t>(c0 + lane) * bs;
    for (int i0 = 0; i0 < bs; i0 += 8) {
      uint32_t x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = i0 + k < bs ? static_cast<uint32_t>(__ldg(t + i0 + k)) : 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (i0 + k < bs) a = a * kHashBase + (static_cast<uint64_t>(x[k]) + 1ull);
    }
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

// The same comparison for a node another warp of the running launch may have written: the node's
// tokens are read through L2 (a read-only-cache line could predate the write).
__device__ __forceinline__ bool block_tokens_equal_coherent(const int32_t* a, const int32_t* node_tok, int bs) {
  int i = 0;
  for (; i + 8 <= bs; i += 8) {
    int32_t x[8], y[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x[k] = __ldg(a + i + k);
      y[k] = __ldcg(node_tok + i + k);
    }
    bool eq = true;
#pragma unroll
    for (int k = 0; k < 8; ++k) eq &= x[k] == y[k];
    if (!eq) return false;
  }
  bool eq = true;
  for (; i < bs; ++i) eq &= __ldg(a + i) == __ldcg(node_tok + i);
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
// One block's step of an ordered walk, run by a whole warp (lane 0 does the atomics), with its probe
// starting at `slot`: an empty slot is claimed with a compare-and-swap and the sequence's own block
// becomes the node (data written, then the slot published); a slot with the same key is waited for
// until published (bounded) and reused when depth, parent and tokens match. Every other slot is
// skipped. Returns the node that holds the block's prefix, or -1 after setting the error bit (no free
// slot, or the wait ran out).
__device__ int insert_step(const PrefixArgs& a, uint64_t key, uint64_t slot, int own, int j, const int32_t* tok,
                           int parent, int lane) {
  const uint64_t mask = static_cast<uint64_t>(a.cap) - 1;
  for (int64_t it = 0; it < a.cap; ++it) {
    uint64_t k = 0;
    // one compare-and-swap both reads the slot and, when it is empty, claims it (0 comes back)
    if (lane == 0) k = atomicCAS(reinterpret_cast<unsigned long long*>(a.slot_keys + slot), 0ull, key);
    k = shfl_u64(k, 0);
    if (k == 0ull) {
      for (int i = lane; i < a.bs; i += 32) a.node_tokens[static_cast<int64_t>(own) * a.bs + i] = __ldg(tok + i);
      if (lane == 0) {
        a.node_parent[own] = parent;
        a.node_depth[own] = j;
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicExch(a.slot_nodes + slot, own);
      return own;
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
        return -1;
      }
      __threadfence();
      bool same = nd < a.num_blocks && __ldcg(a.node_depth + nd) == j && __ldcg(a.node_parent + nd) == parent;
      if (same) {
        bool eq = true;
        for (int i = lane; i < a.bs; i += 32) eq &= (__ldg(tok + i) == __ldcg(a.node_tokens + static_cast<int64_t>(nd) * a.bs + i));
        same = __all_sync(0xffffffffu, eq);
      }
      if (same) return nd;
    }
    slot = (slot + 1) & mask;
  }
  if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_TABLE_FULL);
  return -1;
}

// One warp per sequence, 32 full blocks per round (lane = block):
//   1. Every block of the round claims an empty slot on its key's probe chain with a compare-and-swap,
//      or stops at a slot that already holds its key. Nothing waits here, because the holder of that
//      key (another sequence) may itself still be waiting for this one's earlier blocks.
//   2. The blocks are then resolved in order. A run of claimed blocks is settled at once: each one's
//      node is its own block and its parent the block before it, so the run writes its nodes, fences
//      and publishes them together. A run of blocks that found their keys taken waits for those nodes
//      together and keeps them up to the first that is not its block's prefix; that block then takes
//      one step of the ordered walk (insert_step) from the next slot on.
// The lowest pending block of any sequence can always go on (its parent is settled), so no wait cycle
// forms. Bad block ids are found before any claim, and the walk ends at the first of them. If the walk
// ends early (no free slot, a wait that ran out), the round's claims it did not reach are published as
// node id NB, which no probe accepts, so that nobody waits for them.
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
  int prev = -1;
  int done = 0;
  bool stop = false;
  for (int c0 = 0; c0 < nfull && !stop; c0 += 32) {
    const int count = nfull - c0 < 32 ? nfull - c0 : 32;
    const uint64_t key = chunk_keys(seq, c0, count, a.bs, base_bs, carry, lane);
    const int j = c0 + lane;
    const int own = lane < count ? __ldg(table + j) : 0;
    const uint32_t bad = __ballot_sync(0xffffffffu, lane < count && (own < 0 || own >= a.num_blocks));
    int cnt = count;
    if (bad) {
      cnt = __ffs(bad) - 1;
      stop = true;
      if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_BLOCK_ID);
    }
    // 1. claims
    uint64_t slot = key & mask;
    int state = 0;  // 1 claimed, 2 found its key in a slot, 3 no free slot on the chain
    if (lane < cnt) {
      for (int64_t it = 0; it < a.cap; ++it) {
        const uint64_t k = atomicCAS(reinterpret_cast<unsigned long long*>(a.slot_keys + slot), 0ull, key);
        if (k == 0ull) {
          state = 1;
          break;
        }
        if (k == key) {
          state = 2;
          break;
        }
        slot = (slot + 1) & mask;
      }
      if (state == 0) state = 3;
    }
    // 2. resolution in block order
    const uint32_t claimed = __ballot_sync(0xffffffffu, state == 1);
    const int own_before = __shfl_up_sync(0xffffffffu, own, 1);
    int r = 0;
    while (r < cnt) {
      const uint32_t rest = claimed >> r;
      int run = rest == 0xffffffffu ? 32 : __ffs(~rest) - 1;
      if (run > cnt - r) run = cnt - r;
      if (run > 0) {
        if (lane >= r && lane < r + run) {
          const int32_t* tok = seq + static_cast<int64_t>(j) * a.bs;
          int32_t* dst = a.node_tokens + static_cast<int64_t>(own) * a.bs;
          for (int i0 = 0; i0 < a.bs; i0 += 8) {  // eight loads in flight before their stores
            int32_t x[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = i0 + k < a.bs ? __ldg(tok + i0 + k) : 0;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              if (i0 + k < a.bs) dst[i0 + k] = x[k];
          }
          a.node_parent[own] = lane == r ? prev : own_before;
          a.node_depth[own] = j;
          __threadfence();
          atomicExch(a.slot_nodes + slot, own);
          out[j] = own;
        }
        prev = __shfl_sync(0xffffffffu, own, r + run - 1);
        r += run;
        continue;
      }
      // consecutive blocks from r that found their key: each waits for that slot's node (bounded) and
      // checks it, all at once; a node is this block's prefix when depth, tokens and parent (the node of
      // the block before) match, and the run is taken up to its first block that does not
      const uint32_t held = __ballot_sync(0xffffffffu, state == 2) >> r;
      int hrun = held == 0xffffffffu ? 32 : __ffs(~held) - 1;
      if (hrun > cnt - r) hrun = cnt - r;
      uint64_t from = shfl_u64(slot, r);  // where block r's own step starts
      if (hrun > 0) {
        const bool in = lane >= r && lane < r + hrun;
        int nd = -1, par = -2;
        bool same = false;
        if (in) {
          for (int spin = 0; spin < kSpinLimit; ++spin) {
            nd = atomicAdd(a.slot_nodes + slot, 0);
            if (nd >= 0) break;
            __nanosleep(32);
          }
          if (nd >= 0 && nd < a.num_blocks) {
            __threadfence();
            same = __ldcg(a.node_depth + nd) == j &&
                   block_tokens_equal_coherent(seq + static_cast<int64_t>(j) * a.bs,
                                               a.node_tokens + static_cast<int64_t>(nd) * a.bs, a.bs);
            par = __ldcg(a.node_parent + nd);
          }
        }
        const int nd_before = __shfl_up_sync(0xffffffffu, nd, 1);
        same = same && par == (lane == r ? prev : nd_before);
        const uint32_t ok = __ballot_sync(0xffffffffu, in && same) >> r;
        int good = ok == 0xffffffffu ? 32 : __ffs(~ok) - 1;
        if (good > hrun) good = hrun;
        if (lane >= r && lane < r + good) out[j] = nd;
        if (good > 0) {
          prev = __shfl_sync(0xffffffffu, nd, r + good - 1);
          r += good;
          continue;
        }
        // block r's node is not its prefix (another prefix with the same key) or never came: its own
        // ordered step, from the slot after (or, after a wait that ran out, at) the one it found
        const int nd_r = __shfl_sync(0xffffffffu, nd, r);
        if (nd_r < 0) {
          if (lane == 0) atomicOr(a.error_word, TACO_DEVERR_WAIT_TIMEOUT);
          stop = true;
          break;
        }
        from = (from + 1) & mask;
      }
      const int found = insert_step(a, shfl_u64(key, r), from, __shfl_sync(0xffffffffu, own, r), c0 + r,
                                    seq + static_cast<int64_t>(c0 + r) * a.bs, prev, lane);
      if (found < 0) {
        stop = true;
        break;
      }
      if (lane == 0) out[c0 + r] = found;
      prev = found;
      ++r;
    }
    if (r < cnt && lane >= r && lane < cnt && state == 1) atomicExch(a.slot_nodes + slot, a.num_blocks);
    done = c0 + r;
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
