// Device-side building blocks shared by the verify and append kernels: shared-memory mbarriers,
// TMA tile loads, ldmatrix / mma.sync wrappers, bounded waits and the split-KV work schedule.
#pragma once

#include <cuda.h>
#include <float.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "taco_attn.h"

namespace taco {

constexpr int kTileKeys = 64;                 // keys per pipeline stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a pipeline wait gives up after 2 s
// default L2 prefetch distances (key tiles past the latest load) of the two verify kernels
constexpr int kTcPrefetchTiles = 0;
constexpr int kMmaPrefetchTiles = 0;
// Default segment cost of the work split (see the schedule below), in key tiles of the kernel, from
// the packed query rows of a unit: starting and finishing a segment (query load, epilogue, partial
// write and merge) grows with the rows, a tile's load time does not. Measured best on B200: 2 for
// 8-row and 5 for 32-row units on the mma.sync kernel (64-key tiles), 2-3 for 64-row and 3-5 for
// 128-row units on the tcgen05 kernel (128-key tiles). With e4m3 caches a tcgen05 tile takes about
// one and a half times as long (the softmax warps widen it), so a segment costs fewer tiles: 1
// measured best on chain and tree (2 the same, 0 and 3 slower).
inline int mma_seg_cost(int rows) { return 1 + rows / 8; }
inline int tc_seg_cost(int rows, bool kv8) { return kv8 ? 1 : 1 + rows / 64; }

struct VerifyParams {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* num_candidates;
  const uint32_t* tree_mask_bits;
  float* part_o;         // [slots, rows_per_unit, D] fp32 split-KV partial outputs (normalised)
  float* part_lse;       // [slots, rows_per_unit] base-2 log-sum-exp of each partial
  uint32_t* counters;    // [units] arrivals of split units (zero between calls)
  uint32_t* error_word;  // device error bits
  float scale_log2;      // scale * log2(e)
  int B, C, Hq, Hkv, G, D, bs, num_blocks, max_blocks;
  int rows_per_unit;     // packed query rows handled by one unit (row group)
  int row_groups;        // number of row groups per (sequence, KV head)
  int cands_per_group;   // tensor-core path: candidates per row group (rows = cands_per_group * G)
  int tile_keys;         // keys per work tile of the kernel (64 or 128)
  int l2_prefetch_tiles; // key tiles whose K/V the producer asks L2 to fetch ahead of its loads (0 = none)
  const float* k_scale;  // e4m3 caches: per-KV-head scales (K value = code * k_scale[h]); else null
  const float* v_scale;
  const float* q_scale;  // e4m3 caches on the tcgen05 path: the f16 query rows' scale per row, or null
  // test knobs of the mma.sync kernel (zero = off): a pipeline wait gives up after wait_limit_ns
  // (0 = kWaitLimitNs); with stall_tile = t + 1, CTA 0's producers leave tile t's stage unarmed, so
  // that a consumer's bounded wait runs out
  uint64_t wait_limit_ns;
  int stall_tile;
  // 1 when the grid this launch depends on (programmatic launch) is this library's append kernel with
  // derived slots, launched by the same call: it writes only cache slots [L_b - C, L_b) of each
  // sequence, and everything else the verify reads was complete before it started. The producers then
  // wait for it only before loading a tile that reaches key L_b - C, instead of at the start.
  int late_wait;
  int seg_cost;          // virtual tiles per unit in the work split (see the schedule below); 0 = equal split
  // 1: split units only write their partials (no arrival counting, no merge); the combine kernel run
  // after the verify merges them (mma.sync kernel only)
  int defer_merge;
  // fused append (16-bit caches, units of <= 16 rows): candidate i's new K/V rows [B, C, Hkv, D] go to
  // logical slot P_b + i of these caches as the verify reads them; null = the caches are complete
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
};

// ---------------------------------------------------------------------------------------------
// small PTX wrappers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Non-blocking test of phase completion.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Test for phase completion, suspending up to about `hint_ns` if it is not complete yet.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete. Gives up after limit_ns (kWaitLimitNs when
// 0), sets the timeout bit in the error word and returns false (the caller then leaves its loop).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t* error_word,
                                          uint64_t limit_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = limit_ns ? limit_ns : kWaitLimitNs;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_timer_ns() - t0 > limit) break;
  }
  atomicOr(error_word, TACO_DEVERR_WAIT_TIMEOUT);
  return false;
}

// 2-D TMA tile load global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// L2 prefetch of one TMA tile: no shared memory, no completion. The later tile load of the same
// coordinates then finds its lines in L2 (or already on their way), so HBM latency is covered by
// requests that hold no shared-memory stage.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch. A kernel launched with programmatic stream serialization may start
// while the previous kernel in the stream still runs; grid_dependency_wait() blocks until every grid
// it depends on has completed and its memory is visible (immediately when there is none).
// grid_launch_dependents() lets the next programmatic launch start early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Two e4m3 codes (low byte first) as an f16x2 MMA operand pair (exact: every e4m3 value is an f16
// normal or zero).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t h;
  const uint16_t v = static_cast<uint16_t>(two_codes & 0xffffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return h;
}

// e4m3 of two floats (first in the low byte), round to nearest even, saturating at +-448
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float first, float second) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
  return r;
}

template <typename T>
__device__ __forceinline__ float elt_to_f32(T x);
template <>
__device__ __forceinline__ float elt_to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float elt_to_f32<__half>(__half x) {
  return __half2float(x);
}

// The quantising append's arithmetic on 8 values (one 16-byte piece of a 16-bit row): each value
// divided by the KV head's scale (float32, correctly rounded), then rounded to e4m3; 8 codes, the
// first value's in the lowest byte.
template <typename T>
__device__ __forceinline__ uint2 quantise_e4m3x8(uint4 in, float scale) {
  const T* e = reinterpret_cast<const T*>(&in);
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = f32x2_to_e4m3x2(__fdiv_rn(elt_to_f32<T>(e[2 * i]), scale), __fdiv_rn(elt_to_f32<T>(e[2 * i + 1]), scale));
  return make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// byte permute: bytes 0-3 of a, then 4-7 of b, picked by the four selector nibbles
__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

template <typename T>
struct MmaOp;

template <>
struct MmaOp<__nv_bfloat16> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

template <>
struct MmaOp<__half> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

// ---------------------------------------------------------------------------------------------
// split-KV work schedule ("stream-K" over key tiles)
//
// Work unit u = (b, kv head g, row group rg), ordered u = (b * Hkv + g) * RG + rg. Unit u holds
// T_b = max(1, ceil(L_b / tile_keys)) key tiles (an empty sequence still gets one tile, which
// writes its zero rows). All units' tiles are concatenated into one range of real tiles [0, Wr).
// The split between CTAs is made in a weighted copy of that range: unit u there spans seg_cost
// virtual tiles (the cost of starting and finishing a segment: loading Q, the epilogue, the arrival)
// followed by its T_b real tiles, so it starts at weight S_u = (first real tile of u) + seg_cost * u
// and the total is W = Wr + seg_cost * units. CTA c of the nC working CTAs takes the weights
// [c*W/nC, (c+1)*W/nC), that is the real tiles from the first one at or after weight c*W/nC up to
// the first one at or after (c+1)*W/nC. A CTA whose range crosses many unit starts thus gets fewer
// real tiles; seg_cost = 0 is the plain equal split. A unit that falls into several CTAs' ranges is
// split: each piece writes a partial (normalised output + log-sum-exp), and the CTA that arrives
// last on the unit's counter combines them. Since each CTA's range is contiguous, only its first
// and last piece can be partial, so CTA c owns two partial slots: 2c (its first piece) and 2c+1.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ int clamp_context_value(const VerifyParams& p, int L, bool report) {
  const int cap = p.max_blocks * p.bs;
  if (L < 0 || L > cap) {
    if (report) atomicOr(p.error_word, TACO_DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

__device__ __forceinline__ int clamp_context(const VerifyParams& p, int b, bool report) {
  return clamp_context_value(p, __ldg(p.context_lens + b), report);
}

__device__ __forceinline__ int clamp_candidates_value(const VerifyParams& p, int n, int L, bool report) {
  const int cap = L < p.C ? L : p.C;
  if (n < 0 || n > cap) {
    if (report) atomicOr(p.error_word, TACO_DEVERR_NUM_CAND);
    n = n < 0 ? 0 : cap;
  }
  return n;
}

__device__ __forceinline__ int clamp_candidates(const VerifyParams& p, int b, int L, bool report) {
  return clamp_candidates_value(p, __ldg(p.num_candidates + b), L, report);
}

__device__ __forceinline__ int tiles_of(int L, int tile) { return L <= 0 ? 1 : (L + tile - 1) / tile; }

// the CTA (of nC over total weight W) whose weight range contains weight w
__device__ __forceinline__ int cta_of_tile(int64_t w, int64_t W, int64_t nC) {
  return static_cast<int>(((w + 1) * nC - 1) / W);
}

// The CTAs holding the first and the last real tile of unit u (global ordinal), whose first real
// tile is unit_base and which has Tb tiles, and whether the first of them reaches the unit from an
// earlier unit (then the unit's piece is in its second partial slot).
struct UnitCtas {
  int c_first, c_last;
  bool first_odd;
};
__device__ __forceinline__ UnitCtas unit_ctas(const VerifyParams& p, int64_t unit_base, int Tb, int64_t u,
                                              int64_t W, int nC) {
  const int64_t S = unit_base + static_cast<int64_t>(p.seg_cost) * u;  // weight where the unit starts
  UnitCtas r;
  r.c_first = cta_of_tile(S + p.seg_cost, W, nC);
  r.c_last = cta_of_tile(S + p.seg_cost + Tb - 1, W, nC);
  r.first_odd = static_cast<int64_t>(r.c_first) * W / nC < S;
  return r;
}

struct SchedStart {
  int64_t W;        // total weight (real tiles + seg_cost per unit)
  int nC;           // working CTAs
  int64_t lo, hi;   // this CTA's range of real tiles
  int b;            // sequence of the first unit
  int64_t base_b;   // first tile of sequence b's units
};

// The first real tile at or after weight A (< W), with the sequence holding it and that sequence's
// first tile. Computed by one full warp; every lane returns the same values.
struct SchedPoint {
  int64_t t;
  int b;
  int64_t base_b;
};
__device__ __forceinline__ SchedPoint schedule_locate(const VerifyParams& p, int64_t A) {
  const int lane = threadIdx.x & 31;
  const int HR = p.Hkv * p.row_groups;
  const int c = p.seg_cost;
  int64_t run_w = 0, run_r = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const int Tb = b < p.B ? tiles_of(clamp_context(p, b, false), p.tile_keys) : 0;
    const int64_t mine_r = static_cast<int64_t>(Tb) * HR;
    const int64_t mine_w = b < p.B ? static_cast<int64_t>(Tb + c) * HR : 0;
    int64_t incl_r = mine_r, incl_w = mine_w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t vr = __shfl_up_sync(0xffffffffu, incl_r, o);
      const int64_t vw = __shfl_up_sync(0xffffffffu, incl_w, o);
      if (lane >= o) {
        incl_r += vr;
        incl_w += vw;
      }
    }
    const int64_t excl_w = run_w + incl_w - mine_w;
    const int64_t excl_r = run_r + incl_r - mine_r;
    const bool here = b < p.B && excl_w <= A && A < run_w + incl_w;
    const uint32_t ball = __ballot_sync(0xffffffffu, here);
    if (ball) {
      const int src = __ffs(ball) - 1;
      SchedPoint r;
      r.b = b0 + src;
      r.base_b = __shfl_sync(0xffffffffu, excl_r, src);
      const int64_t off = A - __shfl_sync(0xffffffffu, excl_w, src);  // weight offset into sequence b
      const int T = __shfl_sync(0xffffffffu, Tb, src);
      const int64_t jj = off / (T + c), in = off % (T + c);
      r.t = r.base_b + jj * T + (in > c ? in - c : 0);
      return r;
    }
    run_w += __shfl_sync(0xffffffffu, incl_w, 31);
    run_r += __shfl_sync(0xffffffffu, incl_r, 31);
  }
  SchedPoint r;  // A at or past the end
  r.t = run_r;
  r.b = p.B;
  r.base_b = run_r;
  return r;
}

// Computed by one full warp; every lane returns the same values.
__device__ __forceinline__ SchedStart schedule_start(const VerifyParams& p, int cta, int grid) {
  const int lane = threadIdx.x & 31;
  const int HR = p.Hkv * p.row_groups;
  int64_t Wr = 0;
  for (int b = lane; b < p.B; b += 32) Wr += static_cast<int64_t>(tiles_of(clamp_context(p, b, false), p.tile_keys)) * HR;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Wr += __shfl_xor_sync(0xffffffffu, Wr, o);
  SchedStart s;
  s.W = Wr + static_cast<int64_t>(p.seg_cost) * p.B * HR;
  s.nC = static_cast<int>(Wr < grid ? Wr : grid);
  s.lo = s.hi = 0;
  s.b = 0;
  s.base_b = 0;
  if (cta >= s.nC) return s;
  const SchedPoint a = schedule_locate(p, static_cast<int64_t>(cta) * s.W / s.nC);
  s.lo = a.t;
  s.b = a.b;
  s.base_b = a.base_b;
  s.hi = cta + 1 == s.nC ? Wr : schedule_locate(p, static_cast<int64_t>(cta + 1) * s.W / s.nC).t;
  return s;
}

// Destination of merged row r of a unit: dst == nullptr for a padding row (nothing is written),
// active == false for a row of a padding candidate (written as zeros).
template <typename T>
struct MergeRow {
  T* dst;
  bool active;
};

// Combines the partials of one split unit into its output rows:
//   out_r = sum_s 2^(lse_s,r - M_r) O_s,r / sum_s 2^(lse_s,r - M_r),   M_r = max_s lse_s,r,
// over the pieces s = 0 .. c_last - c_first (CTA order; piece 0 sits in slot 2*c_first + 1 when
// it is not c_first's first segment, every other piece in slot 2c). Partials are stored
// [slot][row (stride rows)][D] fp32 with normalised O, lse in base 2; lse = -inf means the piece
// saw no visible key and weighs 0.
// Run by the 4 warps (wid 0..3) of one 128-thread group. A warp takes 8 rows x 2 pieces per pass,
// with the lse and O loads of the pass all issued before use, so a pass costs one L2 round trip;
// pieces beyond 2 are folded in with an online rescale.
template <typename T, int D, typename RowFn>
__device__ __forceinline__ void merge_split_unit(const VerifyParams& p, int rows, int stride, int c_first,
                                                 int c_last, bool first_odd, int wid, int lane, RowFn row_of) {
  constexpr int RB = 8, SC = 2, V = D / 32;
  static_assert(V == 2 || V == 4, "head_dim 64 or 128");
  const int nsl = c_last - c_first + 1;
  auto slot_of = [&](int s) -> int64_t {
    const int c = c_first + s;
    return (s == 0 && first_odd) ? 2 * c + 1 : 2 * c;
  };
  for (int r0 = wid * RB; r0 < rows; r0 += 4 * RB) {
    float acc[RB][V], m[RB], l[RB];
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      m[k] = -INFINITY;
      l[k] = 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) acc[k][e] = 0.f;
    }
    for (int s0 = 0; s0 < nsl; s0 += SC) {
      float ls = -INFINITY;  // lane j*RB + k holds lse of (piece s0 + j, row r0 + k)
      {
        const int k = lane % RB, j = lane / RB;
        if (j < SC && s0 + j < nsl && r0 + k < rows) ls = __ldcg(p.part_lse + slot_of(s0 + j) * stride + r0 + k);
      }
      float v[SC][RB][V];
#pragma unroll
      for (int j = 0; j < SC; ++j) {
        const bool have = s0 + j < nsl;
        const int64_t sl = have ? slot_of(s0 + j) : 0;
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          if (have && r0 + k < rows) {
            const float* src = p.part_o + (sl * stride + r0 + k) * D + lane * V;
            if constexpr (V == 4) {
              const float4 x = __ldcg(reinterpret_cast<const float4*>(src));
              v[j][k][0] = x.x;
              v[j][k][1] = x.y;
              v[j][k][2] = x.z;
              v[j][k][3] = x.w;
            } else {
              const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
              v[j][k][0] = x.x;
              v[j][k][1] = x.y;
            }
          } else {
#pragma unroll
            for (int e = 0; e < V; ++e) v[j][k][e] = 0.f;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        float lj[SC];
        float cm = m[k];
#pragma unroll
        for (int j = 0; j < SC; ++j) {
          lj[j] = __shfl_sync(0xffffffffu, ls, j * RB + k);
          cm = fmaxf(cm, lj[j]);
        }
        if (cm == -INFINITY) continue;  // nothing visible in this row so far (warp-uniform)
        const float f = m[k] == -INFINITY ? 0.f : exp2f(m[k] - cm);
        l[k] *= f;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[k][e] *= f;
#pragma unroll
        for (int j = 0; j < SC; ++j) {
          if (lj[j] == -INFINITY) continue;
          const float w = exp2f(lj[j] - cm);
          l[k] += w;
#pragma unroll
          for (int e = 0; e < V; ++e) acc[k][e] = fmaf(w, v[j][k][e], acc[k][e]);
        }
        m[k] = cm;
      }
    }
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      if (r0 + k >= rows) break;
      const MergeRow<T> d = row_of(r0 + k);
      if (d.dst == nullptr) continue;
      const float inv = (d.active && l[k] > 0.f) ? 1.f / l[k] : 0.f;
      uint32_t w2[V / 2];
#pragma unroll
      for (int e = 0; e < V / 2; ++e)
        w2[e] = d.active ? MmaOp<T>::pack(acc[k][2 * e] * inv, acc[k][2 * e + 1] * inv) : 0u;
      if constexpr (V == 4)
        *reinterpret_cast<uint2*>(d.dst + lane * V) = make_uint2(w2[0], w2[1]);
      else
        *reinterpret_cast<uint32_t*>(d.dst + lane * V) = w2[0];
    }
  }
}

// Walks one CTA's work as segments: a segment is the part of one unit (b, j = g * RG + rg) that
// falls into the CTA's tile range; tiles [tile, seg_end()) of the unit. The next sequence's context
// length is loaded one sequence ahead, so that moving on does not wait for it.
struct SegCursor {
  int b;
  int64_t base_b;  // first global tile of sequence b's units
  int L, Tb, j, tile;
  int L_next_raw;  // context_lens[b + 1] as loaded (0 past the batch)
  int64_t t, hi;
  int HR;
  int ui;          // segment ordinal within the CTA

  __device__ __forceinline__ void init(const VerifyParams& p, int b0, int64_t base_b0, int64_t lo, int64_t hi_,
                                       bool report) {
    b = b0;
    base_b = base_b0;
    HR = p.Hkv * p.row_groups;
    L = clamp_context(p, b, report);
    L_next_raw = b + 1 < p.B ? __ldg(p.context_lens + b + 1) : 0;
    Tb = tiles_of(L, p.tile_keys);
    t = lo;
    hi = hi_;
    j = static_cast<int>((t - base_b) / Tb);
    tile = static_cast<int>((t - base_b) % Tb);
    ui = 0;
  }
  __device__ __forceinline__ bool valid() const { return t < hi; }
  __device__ __forceinline__ int seg_end() const {
    return static_cast<int>(Tb < tile + (hi - t) ? Tb : tile + (hi - t));
  }
  __device__ __forceinline__ int64_t unit_base() const { return base_b + static_cast<int64_t>(j) * Tb; }
  __device__ __forceinline__ void next_segment(const VerifyParams& p, bool report) {
    t += seg_end() - tile;
    tile = 0;
    ++ui;
    if (++j == HR) {
      j = 0;
      base_b += static_cast<int64_t>(Tb) * HR;
      if (++b < p.B) {
        L = clamp_context_value(p, L_next_raw, report);
        L_next_raw = b + 1 < p.B ? __ldg(p.context_lens + b + 1) : 0;
        Tb = tiles_of(L, p.tile_keys);
      }
    }
  }
};

// Walks a CTA's tiles like its producers do and asks L2 to fetch each tile's K and V chunks, a set
// number of tiles before the producer loads them (tma_prefetch_2d). A shared-memory ring can only
// hold a few tiles while HBM latency under load is several microseconds; these requests keep more of
// the stream in flight without holding any stage. Run by one whole warp; prefetch() issues every tile
// whose CTA-local ordinal is below `upto` and has not been issued yet. Lanes take one chunk each,
// exactly as the loads do, and chunks with a bad block id are skipped (the loads report them).
template <int kPanels, int kColsPerPanel>
struct TilePrefetcher {
  SegCursor c;
  int tl, tend, g, nblk, win;
  int32_t win_val;
  const int32_t* bt_row;
  int64_t next;  // CTA-local ordinal of the next tile to prefetch
  bool have;

  __device__ __forceinline__ void start_segment(const VerifyParams& p) {
    tl = c.tile;
    tend = c.seg_end();
    g = c.j / p.row_groups;
    nblk = (c.L + p.bs - 1) / p.bs;
    bt_row = p.block_tables + static_cast<int64_t>(c.b) * p.max_blocks;
    win = -1000000;
    win_val = -1;
  }
  __device__ __forceinline__ void step(const VerifyParams& p) {
    ++next;
    if (++tl == tend) {
      c.next_segment(p, false);
      have = c.valid();
      if (have) start_segment(p);
    }
  }
  // `skip` leading tiles are passed over (the producer's first loads find an empty ring anyway)
  __device__ __forceinline__ void init(const VerifyParams& p, int b0, int64_t base_b0, int64_t lo, int64_t hi,
                                       int skip) {
    c.init(p, b0, base_b0, lo, hi, false);
    next = 0;
    have = c.valid();
    if (have) start_segment(p);
    while (have && next < skip) step(p);
  }
  __device__ __forceinline__ void prefetch(const VerifyParams& p, int64_t upto, const CUtensorMap* mk,
                                           const CUtensorMap* mv) {
    const int lane = threadIdx.x & 31;
    const int tk = p.tile_keys;
    const int rpc = p.bs < tk ? p.bs : tk;
    const int chunks_per_tile = tk / rpc;
    while (have && next < upto) {
      const int L = c.L;
      const int key0 = tl * tk;
      int nvalid = L > key0 ? (L - key0 + rpc - 1) / rpc : 0;
      if (nvalid > chunks_per_tile) nvalid = chunks_per_tile;
      const int lb_first = key0 / p.bs;
      if (nvalid > 0 && (lb_first < win || (key0 + (nvalid - 1) * rpc) / p.bs >= win + 32)) {
        win = lb_first;
        const int lb = win + lane;
        win_val = lb < nblk ? __ldg(bt_row + lb) : -1;
      }
      const int my_lb = (key0 + lane * rpc) / p.bs;
      const int32_t blk = __shfl_sync(0xffffffffu, win_val, (my_lb - win) & 31);
      if (lane < nvalid && blk >= 0 && blk < p.num_blocks) {
        const int row = (blk * p.Hkv + g) * p.bs + (key0 + lane * rpc) % p.bs;
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn) {
          tma_prefetch_2d(mk, pn * kColsPerPanel, row);
          tma_prefetch_2d(mv, pn * kColsPerPanel, row);
        }
      }
      __syncwarp();
      step(p);
    }
  }
};

// A producer's walk over its CTA's tiles, one tile at a time, with the block-table window of the
// current segment; chunk() gives a lane's chunk of the current tile the way the 16-bit producers
// compute it (lane l takes rows [l rpc, (l + 1) rpc) of the tile; chunks past the context or with a
// bad block id are not loaded).
struct TileLoadCursor {
  SegCursor c;
  int tl, tend, g, nblk, win;
  int32_t win_val;
  const int32_t* bt_row;
  int64_t k;  // CTA-local ordinal of the current tile
  bool have, report;

  __device__ __forceinline__ void start_segment(const VerifyParams& p) {
    tl = c.tile;
    tend = c.seg_end();
    g = c.j / p.row_groups;
    nblk = (c.L + p.bs - 1) / p.bs;
    bt_row = p.block_tables + static_cast<int64_t>(c.b) * p.max_blocks;
    win = -1000000;
    win_val = -1;
  }
  __device__ __forceinline__ void init(const VerifyParams& p, int b0, int64_t base_b0, int64_t lo, int64_t hi,
                                       bool report_) {
    report = report_;
    c.init(p, b0, base_b0, lo, hi, report);
    k = 0;
    have = c.valid();
    if (have) start_segment(p);
  }
  __device__ __forceinline__ void step(const VerifyParams& p) {
    ++k;
    if (++tl == tend) {
      c.next_segment(p, report);
      have = c.valid();
      if (have) start_segment(p);
    }
  }
  // Whole warp. Returns whether this lane loads a chunk; *row is its first cache row, *nloaded the
  // number of chunks the warp loads.
  __device__ __forceinline__ bool chunk(const VerifyParams& p, int tk, int rpc, int* row, int* nloaded) {
    const int lane = threadIdx.x & 31;
    const int chunks_per_tile = tk / rpc;
    const int L = c.L;
    const int key0 = tl * tk;
    int nvalid = L > key0 ? (L - key0 + rpc - 1) / rpc : 0;
    if (nvalid > chunks_per_tile) nvalid = chunks_per_tile;
    const int lb_first = key0 / p.bs;
    if (nvalid > 0 && (lb_first < win || (key0 + (nvalid - 1) * rpc) / p.bs >= win + 32)) {
      win = lb_first;
      const int lb = win + lane;
      win_val = lb < nblk ? __ldg(bt_row + lb) : -1;
    }
    const int my_lb = (key0 + lane * rpc) / p.bs;
    const int32_t blk = __shfl_sync(0xffffffffu, win_val, (my_lb - win) & 31);
    bool ok = lane < nvalid;
    if (ok && (blk < 0 || blk >= p.num_blocks)) {
      if (report) atomicOr(p.error_word, TACO_DEVERR_BLOCK_ID);
      ok = false;
    }
    *nloaded = __popc(__ballot_sync(0xffffffffu, ok));
    *row = (blk * p.Hkv + g) * p.bs + (key0 + lane * rpc) % p.bs;
    return ok;
  }
};

struct TileInfo {
  int b, j;    // the tile's sequence and unit within it (j = kv head * row groups + row group)
  int ui;      // segment ordinal within the CTA
  int tl;      // tile index within the unit
  int jl;      // tile index within the segment
  bool first;  // first tile of its segment
  bool last;   // last tile of its segment
};

// Tile-by-tile walk over the same sequence of segments.
struct TileWalker {
  SegCursor c;
  int tl, tend;
  bool have;
  __device__ __forceinline__ void init(const VerifyParams& p, int b0, int64_t base_b0, int64_t lo, int64_t hi) {
    c.init(p, b0, base_b0, lo, hi, false);
    have = c.valid();
    if (have) {
      tl = c.tile;
      tend = c.seg_end();
    }
  }
  __device__ __forceinline__ bool next(const VerifyParams& p, TileInfo& ti) {
    if (!have) return false;
    ti.b = c.b;
    ti.j = c.j;
    ti.ui = c.ui;
    ti.tl = tl;
    ti.jl = tl - c.tile;
    ti.first = (tl == c.tile);
    ti.last = (tl == tend - 1);
    if (++tl == tend) {
      c.next_segment(p, false);
      have = c.valid();
      if (have) {
        tl = c.tile;
        tend = c.seg_end();
      }
    }
    return true;
  }
};

}  // namespace taco
