// Verify kernel for narrow packed query tiles (G * C up to 64 rows per unit): the warp-level
// mma.sync path.
//
// One CTA = 4 consumer warps + 2 producer warps, two CTAs per SM, persistent over a stream-K range of
// key tiles (device_common.cuh). The producer warps walk the block table and stream each tile's
// K chunks (first producer) and V chunks (second producer) (one chunk = min(bs, tile) consecutive
// slots of one physical block and one KV head, contiguous in the [NB, Hkv, bs, D] cache) into a ring
// of shared-memory stages with TMA, 128-byte swizzled so that ldmatrix reads are conflict-free. A
// single warp can keep only so many TMA copies moving, so K and V are issued from separate warps;
// both walk every stage in order and arm the stage's full barrier (arrival count 2). Consumer warps own 16 packed query rows each
// (rows r = i * G + h' of candidate i and head g*G + h') and, when fewer than 4 row tiles exist,
// split the tile's keys between them; S = Q K^T and O += P V run on mma.sync m16n8k16 with fp32
// accumulators, and the softmax is the flash-style online form in base 2 (fp32 running max / sum).
// The tree mask only enters the tiles that reach the candidates' positions. Units of at most 8 rows
// use the swapped form (S^T = K Q^T, see MmaCfg), and e4m3 caches a variant that widens the codes to
// f16 in registers (KV8).
#pragma once

#include "device_common.cuh"

namespace taco {

// MT = number of 16-row query tiles per unit (1, 2, 4), or 0 for the swapped form used for units of at
// most 8 packed rows: S^T = K Q^T and O^T = V^T P^T, keys and head dims on the MMA's 16-row side and
// the 8 query rows on its 8-column side, so that no MMA row is spent on padding queries.
template <int D, int MT, bool KV8 = false>
struct MmaCfg {
  static constexpr bool kSwap = (MT == 0);
  static constexpr int kConsumerWarps = 4;
  static constexpr int kProducerWarps = 2;                   // K and V
  static constexpr int kThreads = (kConsumerWarps + kProducerWarps) * 32;
  static constexpr int KG = kSwap ? kConsumerWarps : kConsumerWarps / MT;   // key groups
  // keys per tile: e4m3 tiles carry half the bytes per key, so narrow units take 128 keys per tile
  // to keep the per-tile work (and its fixed costs) in proportion to the bytes it brings
  static constexpr int kTile = (KV8 && MT <= 2) ? 128 : kTileKeys;
  static constexpr int kKeysPerWarp = kTile / KG;             // 16 .. 64
  static constexpr int kRows = kSwap ? 8 : 16 * MT;           // packed rows per unit
  // 128-byte-wide column panels of a K or V row: 64 16-bit values, or 128 e4m3 codes (KV8)
  static constexpr int kColsPerPanel = KV8 ? 128 : 64;
  static constexpr int kPanels = D / kColsPerPanel;
  static constexpr int kPanelBytes = kTile * 128;
  static constexpr int kTensorBytes = kPanels * kPanelBytes;  // one of K or V per stage
  static constexpr int kStageBytes = 2 * kTensorBytes;
  // two CTAs per SM with 96 KB of stages each (three CTAs with 64 KB each and threads capped at 112
  // registers measured slower for the swapped form: the cap spills inside the tile loop)
  static constexpr int kCtasPerSm = 2;
  static constexpr int kStages = 98304 / kStageBytes;
  static constexpr int kScratchFloats = 16 * D + 64;          // cross-warp O and l
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes +
                                    kScratchFloats * 4 + 64 * 4 /*m publish*/ +
                                    2 * kStages * 8 /*barriers*/ + 64 /*schedule*/;
};

struct SchedShared {
  long long W, lo, hi, base_b;
  int nC, b, merge_flag, abort_flag;
};

// e4m3 caches: a query row (16 words of two values per thread, 4 threads per row, neighbouring lanes)
// as f16 pairs. bf16 rows are multiplied by the power of two 2^k that puts the row's largest magnitude
// in [2^14, 2^15) (exact for every element down to 2^-29 of it); returns 2^-k, which the logit scale
// takes. f16 rows are used as they are.
template <typename T>
__device__ __forceinline__ float q_row_to_f16(uint32_t (&w)[16]) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    float mx = 0.f;
#pragma unroll
    for (int v = 0; v < 16; ++v)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[v] << 16)), fabsf(__uint_as_float(w[v] & 0xffff0000u))));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    int k = 0;
    if (mx > 0.f && mx <= FLT_MAX) {
      const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;
      k = 14 - e < 64 ? 14 - e : 64;
    }
    const float up = __uint_as_float(static_cast<uint32_t>(127 + k) << 23);
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const __half2 hv = __floats2half2_rn(__uint_as_float(w[v] << 16) * up, __uint_as_float(w[v] & 0xffff0000u) * up);
      w[v] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    return __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
  } else {
    return 1.f;
  }
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <typename T, int D, int MT, bool KV8>
__global__ void __launch_bounds__(MmaCfg<D, MT>::kThreads, MmaCfg<D, MT>::kCtasPerSm)
    verify_mma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const VerifyParams p) {
  using Cfg = MmaCfg<D, MT, KV8>;
  using Op = MmaOp<T>;
  // e4m3 caches: every product runs as f16 x f16 (K and V codes widen exactly to f16)
  using MOp = typename std::conditional<KV8, MmaOp<__half>, MmaOp<T>>::type;
  constexpr int KG = Cfg::KG;
  constexpr int KW = Cfg::kKeysPerWarp;
  constexpr int NT = KW / 8;          // 8-key n-tiles per warp and tile
  constexpr int DT = D / 8;           // 8-wide d tiles of the output
  constexpr int KSTEPS = D / 16;      // k steps of Q K^T
  constexpr int ROWS = Cfg::kRows;
  constexpr bool SW = Cfg::kSwap;
  constexpr int MTS = SW ? 1 : MT;     // query row tiles (the swapped form has one of 8 rows)
  constexpr int NM = KW / 16;         // swapped form: 16-key m tiles per warp and tile
  constexpr int OT = SW ? D / 16 : DT;   // output accumulator tiles (16 head dims x 8 rows when swapped)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* scratch = reinterpret_cast<float*>(smem + Cfg::kStages * Cfg::kStageBytes);
  float* scratch_l = scratch + 16 * D;
  float* m_pub = scratch + Cfg::kScratchFloats;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(m_pub + 64);
  uint64_t* empty_bar = full_bar + Cfg::kStages;
  SchedShared* sched = reinterpret_cast<SchedShared*>(empty_bar + Cfg::kStages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int HR = p.Hkv * p.row_groups;

  if (tid == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(smem_addr(full_bar + s), Cfg::kProducerWarps);
      mbar_init(smem_addr(empty_bar + s), Cfg::kConsumerWarps);
    }
    fence_mbar_init();
  }
  // inputs (and the cache an append just wrote) are read only after the grids this launch depends on;
  // after this library's own append only the producers wait, before the tiles that hold its slots
  if (!p.late_wait) grid_dependency_wait();
  if (warp == Cfg::kConsumerWarps) {
    SchedStart s = schedule_start(p, blockIdx.x, gridDim.x);
    if (lane == 0) {
      sched->W = s.W;
      sched->lo = s.lo;
      sched->hi = s.hi;
      sched->base_b = s.base_b;
      sched->nC = s.nC;
      sched->b = s.b;
      sched->merge_flag = 0;
      sched->abort_flag = 0;
    }
  }
  __syncthreads();
  const int64_t W = sched->W;
  const int nC = sched->nC;
  if (static_cast<int>(blockIdx.x) >= nC) return;
  const int64_t lo = sched->lo, hi = sched->hi;
  volatile int* abort_flag = &sched->abort_flag;

  if (warp >= Cfg::kConsumerWarps) {
    // ------------------------------------------------------------------ producer warps (K, V)
    const bool is_k = (warp == Cfg::kConsumerWarps);
    const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
    prefetch_tensormap(tmap);
    const uint64_t policy = policy_evict_first();
    const int rpc = p.bs < Cfg::kTile ? p.bs : Cfg::kTile;   // rows per chunk
    const int chunks_per_tile = Cfg::kTile / rpc;
    const uint32_t chunk_bytes = static_cast<uint32_t>(rpc) * 128u;
    int stage = 0;
    uint32_t phase = 0;
    int b = sched->b;
    int64_t base_b = sched->base_b;
    int L = clamp_context(p, b, is_k);
    int Tb = tiles_of(L, Cfg::kTile);
    int64_t t = lo;
    int j = static_cast<int>((t - base_b) / Tb);
    int tile = static_cast<int>((t - base_b) % Tb);
    // the V producer also asks L2 for both tensors of the tile pf_ahead tiles past its latest load
    const int pf_ahead = is_k ? 0 : p.l2_prefetch_tiles;
    TilePrefetcher<Cfg::kPanels, Cfg::kColsPerPanel> pf;
    if (pf_ahead > 0) pf.init(p, b, base_b, lo, hi, Cfg::kStages);
    int64_t kt = 0;  // tile ordinal within the CTA
    bool dep_done = !p.late_wait;
    while (t < hi) {
      const int g = j / p.row_groups;
      const int tend = static_cast<int>(Tb < tile + (hi - t) ? Tb : tile + (hi - t));
      const int nblk = (L + p.bs - 1) / p.bs;
      const int32_t* bt_row = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
      int win = -1000000;
      int32_t win_val = -1;
      for (int tl = tile; tl < tend; ++tl) {
        const int key0 = tl * Cfg::kTile;
        int nvalid = L > key0 ? (L - key0 + rpc - 1) / rpc : 0;
        if (nvalid > chunks_per_tile) nvalid = chunks_per_tile;
        // block ids of this tile's chunks (window of 32 logical blocks held one per lane)
        const int lb_first = key0 / p.bs;
        if (nvalid > 0 && (lb_first < win || (key0 + (nvalid - 1) * rpc) / p.bs >= win + 32)) {
          win = lb_first;
          const int lb = win + lane;
          win_val = lb < nblk ? __ldg(bt_row + lb) : -1;
        }
        int my_lb = (key0 + lane * rpc) / p.bs;
        int32_t blk = __shfl_sync(0xffffffffu, win_val, (my_lb - win) & 31);
        bool ok = lane < nvalid;
        if (ok && (blk < 0 || blk >= p.num_blocks)) {
          if (is_k) atomicOr(p.error_word, TACO_DEVERR_BLOCK_ID);
          ok = false;
        }
        const uint32_t okmask = __ballot_sync(0xffffffffu, ok);
        const uint32_t bytes = __popc(okmask) * chunk_bytes * Cfg::kPanels;
        // test knob: both producers of CTA 0 leave this stage unarmed (no arrival, no copy)
        const bool stall = p.stall_tile != 0 && blockIdx.x == 0 && kt == p.stall_tile - 1;
        bool go = true;
        if (lane == 0) {
          go = (*abort_flag == 0) && mbar_wait(smem_addr(empty_bar + stage), phase ^ 1u, p.error_word, p.wait_limit_ns);
          if (!go) *abort_flag = 1;
          if (!stall) mbar_arrive_expect_tx(smem_addr(full_bar + stage), go ? bytes : 0u);
        }
        go = go && !stall;
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!dep_done && key0 + Cfg::kTile > L - p.C) {  // the tile may hold slots the append wrote
          grid_dependency_wait();
          dep_done = true;
        }
        if (go && ok) {
          const uint32_t dst = smem_addr(stages + stage * Cfg::kStageBytes) + (is_k ? 0u : Cfg::kTensorBytes) +
                               lane * chunk_bytes;
          const int row = (blk * p.Hkv + g) * p.bs + (key0 + lane * rpc) % p.bs;
          const uint32_t fb = smem_addr(full_bar + stage);
#pragma unroll
          for (int pn = 0; pn < Cfg::kPanels; ++pn) tma_load_2d(dst + pn * Cfg::kPanelBytes, tmap, fb, pn * Cfg::kColsPerPanel, row, policy);
        }
        __syncwarp();
        ++kt;
        if (go && pf_ahead > 0) pf.prefetch(p, kt + pf_ahead, &tmap_k, &tmap_v);
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      t += tend - tile;
      tile = 0;
      if (++j == HR) {
        j = 0;
        base_b += static_cast<int64_t>(Tb) * HR;
        if (++b < p.B) {
          L = clamp_context(p, b, is_k);
          Tb = tiles_of(L, Cfg::kTile);
        }
      }
    }
    // make sure no copy of ours is still landing when the CTA exits
    if (lane == 0) {
      for (int s = 0; s < Cfg::kStages; ++s) {
        // the most recent use of stage s completed phase (uses-1); waiting for its parity is
        // immediate when it has landed (or when the stage was never used)
        int uses_parity_phase = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait(smem_addr(full_bar + s), static_cast<uint32_t>(uses_parity_phase), p.error_word, p.wait_limit_ns);
      }
    }
    return;
  }

  // -------------------------------------------------------------------- consumer warps
  const int mt = warp % MTS;
  const int kg = warp / MTS;
  const int gq = lane >> 2;
  const int tq = lane & 3;
  int stage = 0;
  uint32_t phase = 0;
  int b = sched->b;
  int64_t base_b = sched->base_b;
  int L = clamp_context(p, b, false);
  int Tb = tiles_of(L, Cfg::kTile);
  int64_t t = lo;
  int j = static_cast<int>((t - base_b) / Tb);
  int tile = static_cast<int>((t - base_b) % Tb);
  bool first_segment = true;

  while (t < hi) {
    const int g = j / p.row_groups;
    // e4m3 caches: the K scale joins the logit scale, the V scale multiplies O when it is written
    const float sl2 = KV8 ? p.scale_log2 * __ldg(p.k_scale + g) : p.scale_log2;
    const float vsc = KV8 ? __ldg(p.v_scale + g) : 1.f;
    const int rg = j % p.row_groups;
    const int tbegin = tile;
    const int tend = static_cast<int>(Tb < tile + (hi - t) ? Tb : tile + (hi - t));
    const int n = clamp_candidates(p, b, L, first_segment && warp == 0 && lane == 0 && tile == 0);
    const int P = L - n;
    const uint32_t nmask = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);

    // this thread's two packed rows
    int Rrow[2];
    bool rvalid[2];
    uint32_t mw[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // swapped form: the thread's S^T columns (queries 2tq, 2tq+1); otherwise rows gq, gq+8
      Rrow[h] = SW ? rg * ROWS + 2 * tq + h : rg * ROWS + mt * 16 + gq + 8 * h;
      rvalid[h] = Rrow[h] < p.G * n;
      mw[h] = rvalid[h] ? (__ldg(p.tree_mask_bits + static_cast<int64_t>(b) * p.C + Rrow[h] / p.G) & nmask) : 0u;
    }
    // Q fragments: the A operand of m16n8k16 (rows gq / gq+8, columns 2*tq.. of each 16-wide k step), or
    // in the swapped form the B operand (query row gq, the same columns)
    uint32_t qf[KSTEPS][SW ? 2 : 4];
    float sl2r[2] = {sl2, sl2};   // logit scale of this thread's two rows / columns (base 2)
    if constexpr (SW) {
      const int Rq = rg * ROWS + gq;
      const bool qv = Rq < p.G * n;
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          static_cast<const T*>(p.q) +
          ((static_cast<int64_t>(b) * p.C + (qv ? Rq / p.G : 0)) * p.Hq + g * p.G + (qv ? Rq % p.G : 0)) * D);
      if constexpr (!KV8) {
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          qf[kk][0] = qv ? __ldg(qr + kk * 8 + tq) : 0u;
          qf[kk][1] = qv ? __ldg(qr + kk * 8 + 4 + tq) : 0u;
        }
      } else {
        // permuted k order (as below): k step kk, pair j takes head dims tq*32 + kk*4 + 2j (+1)
        uint32_t w[16];
        const uint4* q4 = reinterpret_cast<const uint4*>(qr + tq * 16);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = qv ? __ldg(q4 + v) : make_uint4(0u, 0u, 0u, 0u);
          w[4 * v] = x.x;
          w[4 * v + 1] = x.y;
          w[4 * v + 2] = x.z;
          w[4 * v + 3] = x.w;
        }
        const float down = q_row_to_f16<T>(w);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          qf[kk][0] = w[2 * kk];
          qf[kk][1] = w[2 * kk + 1];
        }
        // the scale of query column c sits with the lanes that loaded row c (lane c * 4)
        sl2r[0] = sl2 * __shfl_sync(0xffffffffu, down, (2 * tq) * 4);
        sl2r[1] = sl2 * __shfl_sync(0xffffffffu, down, (2 * tq + 1) * 4);
      }
    } else {
      const uint32_t* qrow[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = Rrow[h] / p.G, hh = Rrow[h] % p.G;
        qrow[h] = reinterpret_cast<const uint32_t*>(static_cast<const T*>(p.q) +
                                                    ((static_cast<int64_t>(b) * p.C + i) * p.Hq + g * p.G + hh) * D);
      }
      if constexpr (!KV8) {
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          qf[kk][0] = rvalid[0] ? __ldg(qrow[0] + kk * 8 + tq) : 0u;
          qf[kk][1] = rvalid[1] ? __ldg(qrow[1] + kk * 8 + tq) : 0u;
          qf[kk][2] = rvalid[0] ? __ldg(qrow[0] + kk * 8 + 4 + tq) : 0u;
          qf[kk][3] = rvalid[1] ? __ldg(qrow[1] + kk * 8 + 4 + tq) : 0u;
        }
      } else {
        // The k order of Q K^T is permuted (the sum does not depend on it) so that a thread's K codes
        // are 32 consecutive bytes of the key row: k step kk, A/B pair j (0: k = 2tq, 2tq+1; 1: k =
        // 2tq+8, 2tq+9) takes head dims tq*32 + kk*4 + 2j (+1).
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w[16];
          const uint4* q4 = reinterpret_cast<const uint4*>(qrow[h] + tq * 16);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 x = rvalid[h] ? __ldg(q4 + v) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * v] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
          }
          sl2r[h] = sl2 * q_row_to_f16<T>(w);
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            qf[kk][h] = w[2 * kk];
            qf[kk][2 + h] = w[2 * kk + 1];
          }
        }
      }
    }
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float o[OT][4];
#pragma unroll
    for (int dt = 0; dt < OT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

    for (int tl = tbegin; tl < tend; ++tl) {
      const int key0 = tl * Cfg::kTile;
      bool ready = false;
      if (*abort_flag == 0) {
        ready = mbar_wait(smem_addr(full_bar + stage), phase, p.error_word, p.wait_limit_ns);
        if (!ready) *abort_flag = 1;
      }
      const uint32_t kbase = smem_addr(stages + stage * Cfg::kStageBytes);
      const uint32_t vbase = kbase + Cfg::kTensorBytes;
      const int wkey0 = kg * KW;   // first tile-relative key of this warp
      if (ready && key0 + Cfg::kTile > L) {
        // keys >= L in this tile: their V rows may be stale or NaN-poisoned; zero this warp's
        int zr0 = L - key0 - wkey0;
        if (zr0 < 0) zr0 = 0;
        uint8_t* vgen = stages + stage * Cfg::kStageBytes + Cfg::kTensorBytes;
        for (int idx = lane; idx < (KW - zr0) * Cfg::kPanels * 8; idx += 32) {
          const int r = wkey0 + zr0 + idx / (Cfg::kPanels * 8);
          const int rem = idx % (Cfg::kPanels * 8);
          *reinterpret_cast<uint4*>(vgen + (rem / 8) * Cfg::kPanelBytes + r * 128 + (rem % 8) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if constexpr (!KV8 && MTS == 1) {
        // fused append: the candidates' keys P .. L-1 that fall in this warp's key range were loaded
        // from cache slots not yet written; put their new K/V rows into the stage (128-byte swizzle)
        // and into the cache slots. One key group per warp and one row group per unit, so each
        // candidate row has exactly one writer in the launch.
        if (ready && p.k_new != nullptr && key0 + Cfg::kTile > P) {
          const int p_lo = key0 + wkey0 > P ? key0 + wkey0 : P;
          const int p_hi = key0 + wkey0 + KW < L ? key0 + wkey0 + KW : L;
          constexpr int CH = D / 8;   // 16-byte chunks per row
          uint8_t* kgen = stages + stage * Cfg::kStageBytes;
          for (int idx = lane; idx < (p_hi - p_lo) * 2 * CH; idx += 32) {
            const int pos = p_lo + idx / (2 * CH);
            const int rem = idx % (2 * CH);
            const bool is_v = rem >= CH;
            const int c = rem % CH;
            const int64_t src_row = (static_cast<int64_t>(b) * p.C + (pos - P)) * p.Hkv + g;
            const uint4 val = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(is_v ? p.v_new : p.k_new) +
                                                                   src_row * D) + c);
            const int r = pos - key0;
            *reinterpret_cast<uint4*>(kgen + (is_v ? Cfg::kTensorBytes : 0) + (c / 8) * Cfg::kPanelBytes + r * 128 +
                                      (((c % 8) ^ (r & 7)) << 4)) = val;
            const int blk = __ldg(p.block_tables + static_cast<int64_t>(b) * p.max_blocks + pos / p.bs);
            if (blk >= 0 && blk < p.num_blocks) {
              T* cache = static_cast<T*>(is_v ? p.v_cache : p.k_cache);
              reinterpret_cast<uint4*>(cache + ((static_cast<int64_t>(blk) * p.Hkv + g) * p.bs + pos % p.bs) * D)[c] = val;
            } else if (c == 0 && !is_v) {
              atomicOr(p.error_word, TACO_DEVERR_BLOCK_ID);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      if constexpr (KV8 && MTS == 1) {
        // fused quantising append (e4m3 caches), the same division of rows between warps: each new
        // K/V row is divided by its KV head's scale and rounded to e4m3 as the append kernel does,
        // 16 codes (two 16-byte pieces of the 16-bit row) per 16-byte chunk of the stage and the cache
        if (ready && p.k_new != nullptr && key0 + Cfg::kTile > P) {
          const int p_lo = key0 + wkey0 > P ? key0 + wkey0 : P;
          const int p_hi = key0 + wkey0 + KW < L ? key0 + wkey0 + KW : L;
          constexpr int CH = D / 16;  // 16-code chunks per row
          const float ksc = __ldg(p.k_scale + g), vscl = __ldg(p.v_scale + g);
          uint8_t* kgen = stages + stage * Cfg::kStageBytes;
          for (int idx = lane; idx < (p_hi - p_lo) * 2 * CH; idx += 32) {
            const int pos = p_lo + idx / (2 * CH);
            const int rem = idx % (2 * CH);
            const bool is_v = rem >= CH;
            const int c = rem % CH;
            const int64_t src_row = (static_cast<int64_t>(b) * p.C + (pos - P)) * p.Hkv + g;
            const uint4* src =
                reinterpret_cast<const uint4*>(static_cast<const T*>(is_v ? p.v_new : p.k_new) + src_row * D) + 2 * c;
            const float sc = is_v ? vscl : ksc;
            const uint2 lo8 = quantise_e4m3x8<T>(__ldg(src), sc);
            const uint2 hi8 = quantise_e4m3x8<T>(__ldg(src + 1), sc);
            const uint4 codes = make_uint4(lo8.x, lo8.y, hi8.x, hi8.y);
            const int r = pos - key0;
            *reinterpret_cast<uint4*>(kgen + (is_v ? Cfg::kTensorBytes : 0) + r * 128 + ((c ^ (r & 7)) << 4)) = codes;
            const int blk = __ldg(p.block_tables + static_cast<int64_t>(b) * p.max_blocks + pos / p.bs);
            if (blk >= 0 && blk < p.num_blocks) {
              uint8_t* cache = static_cast<uint8_t*>(is_v ? p.v_cache : p.k_cache);
              reinterpret_cast<uint4*>(cache + ((static_cast<int64_t>(blk) * p.Hkv + g) * p.bs + pos % p.bs) * D)[c] =
                  codes;
            } else if (c == 0 && !is_v) {
              atomicOr(p.error_word, TACO_DEVERR_BLOCK_ID);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      if (ready) {
        if constexpr (SW) {
          // ---- swapped form. S^T = K Q^T: m tile m holds keys wkey0 + m*16 .. +15 (rows gq, gq+8 of the
          // C fragment) and the 8 query columns (2tq, 2tq+1); even and odd k steps go to separate
          // accumulators to halve the dependent MMA chain.
          float s[NM][4];
          {
            float s2[NM][4];
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int e = 0; e < 4; ++e) s[m][e] = s2[m][e] = 0.f;
            if constexpr (!KV8) {
#pragma unroll
              for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                  // A = K rows (keys x head dims), row-major: the four 8x8 pieces of ldmatrix
                  const int key = wkey0 + m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                  const int d = kk * 16 + (lane >> 4) * 8;
                  const int c = (d & 63) >> 3;
                  const uint32_t addr = kbase + (d >> 6) * Cfg::kPanelBytes + key * 128 + ((c ^ (key & 7)) << 4);
                  uint32_t a[4];
                  ldsm_x4(addr, a[0], a[1], a[2], a[3]);
                  MOp::run((kk & 1) ? s2[m] : s[m], a, qf[kk][0], qf[kk][1]);
                }
              }
            } else {
              // permuted k order: the A pairs of k step kk are word kk of the 32 bytes at head dim tq*32
              // of key rows gq and gq+8 (both with row & 7 == gq)
#pragma unroll
              for (int m = 0; m < NM; ++m) {
                const uint32_t r0 = kbase + (wkey0 + m * 16 + gq) * 128;
                const uint32_t r1 = r0 + 8 * 128;
                const uint32_t c0 = ((2 * tq) ^ gq) << 4, c1 = ((2 * tq + 1) ^ gq) << 4;
                const uint4 x00 = lds_v4(r0 + c0), x01 = lds_v4(r0 + c1);
                const uint4 x10 = lds_v4(r1 + c0), x11 = lds_v4(r1 + c1);
                const uint32_t k0[8] = {x00.x, x00.y, x00.z, x00.w, x01.x, x01.y, x01.z, x01.w};
                const uint32_t k1[8] = {x10.x, x10.y, x10.z, x10.w, x11.x, x11.y, x11.z, x11.w};
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                  uint32_t a[4];
                  a[0] = e4m3x2_to_f16x2(k0[kk]);
                  a[1] = e4m3x2_to_f16x2(k1[kk]);
                  a[2] = e4m3x2_to_f16x2(k0[kk] >> 16);
                  a[3] = e4m3x2_to_f16x2(k1[kk] >> 16);
                  MOp::run((kk & 1) ? s2[m] : s[m], a, qf[kk][0], qf[kk][1]);
                }
              }
            }
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
              for (int e = 0; e < 4; ++e) s[m][e] += s2[m][e];
          }
          // scale, mask (element e: key gq + 8*(e>>1) of the m tile, query column 2tq + (e&1))
          const bool need_mask = key0 + Cfg::kTile > P;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float v = s[m][e] * sl2r[e & 1];
              if (need_mask) {
                const int key = key0 + wkey0 + m * 16 + gq + 8 * (e >> 1);
                const bool vis = key < P || (key < L && ((mw[e & 1] >> ((key - P) & 31)) & 1u));
                v = vis ? v : -INFINITY;
              }
              s[m][e] = v;
            }
          }
          // online softmax per query column: its keys are spread over the 8 lanes of equal tq
          float alpha[2];
#pragma unroll
          for (int jq = 0; jq < 2; ++jq) {
            float mx = -INFINITY;
#pragma unroll
            for (int m = 0; m < NM; ++m) mx = fmaxf(mx, fmaxf(s[m][jq], s[m][2 + jq]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[jq], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            alpha[jq] = fast_exp2(m_run[jq] - m_use);
            m_run[jq] = m_new;
            float rs = 0.f;
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              const float p0 = fast_exp2(s[m][jq] - m_use);
              const float p1 = fast_exp2(s[m][2 + jq] - m_use);
              s[m][jq] = p0;
              s[m][2 + jq] = p1;
              rs += p0 + p1;
            }
            l_run[jq] = l_run[jq] * alpha[jq] + rs;
          }
          if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
            for (int md = 0; md < OT; ++md) {
              o[md][0] *= alpha[0];
              o[md][1] *= alpha[1];
              o[md][2] *= alpha[0];
              o[md][3] *= alpha[1];
            }
          }
          // O^T += V^T P^T, one k step per m tile of S^T. P^T's B fragment is the transpose of the
          // thread's C fragment: pack (keys gq / gq+8 x columns 2tq, 2tq+1) as 8x8 b16 pieces and
          // transpose them across the warp.
#pragma unroll
          for (int ks = 0; ks < NM; ++ks) {
            const uint32_t pb0 = movmatrix_trans(MOp::pack(s[ks][0], s[ks][1]));
            const uint32_t pb1 = movmatrix_trans(MOp::pack(s[ks][2], s[ks][3]));
            if constexpr (!KV8) {
#pragma unroll
              for (int md = 0; md < OT; ++md) {
                // A = V^T (head dims x keys): V rows read transposed; m rows gq / gq+8 are head dims
                // md*16 + gq / + 8
                const int key = wkey0 + ks * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int d = md * 16 + ((lane >> 3) & 1) * 8;
                const int c = (d & 63) >> 3;
                const uint32_t addr = vbase + (d >> 6) * Cfg::kPanelBytes + key * 128 + ((c ^ (key & 7)) << 4);
                uint32_t a[4];
                ldsm_x4_trans(addr, a[0], a[1], a[2], a[3]);
                MOp::run(o[md], a, pb0, pb1);
              }
            } else {
              // permuted head dims: m rows gq / gq+8 of m tile md are head dims gq*16 + md / + 8, so
              // the A pairs are bytes md and 8 + md of chunk gq of key rows 2tq, 2tq+1, 2tq+8, 2tq+9
              const int kr = wkey0 + ks * 16 + 2 * tq;
              const uint4 x0 = lds_v4(vbase + kr * 128 + ((gq ^ (2 * tq)) << 4));
              const uint4 x1 = lds_v4(vbase + (kr + 1) * 128 + ((gq ^ (2 * tq + 1)) << 4));
              const uint4 x2 = lds_v4(vbase + (kr + 8) * 128 + ((gq ^ (2 * tq)) << 4));
              const uint4 x3 = lds_v4(vbase + (kr + 9) * 128 + ((gq ^ (2 * tq + 1)) << 4));
              const uint32_t r0[4] = {x0.x, x0.y, x0.z, x0.w}, r1[4] = {x1.x, x1.y, x1.z, x1.w};
              const uint32_t r2[4] = {x2.x, x2.y, x2.z, x2.w}, r3[4] = {x3.x, x3.y, x3.z, x3.w};
#pragma unroll
              for (int wd = 0; wd < 2; ++wd) {
#pragma unroll
                for (int i = 0; i < 4; i += 2) {
                  const uint32_t sel = i | ((4 + i) << 4) | ((i + 1) << 8) | ((5 + i) << 12);
                  const uint32_t a0 = byte_perm(r0[wd], r1[wd], sel);
                  const uint32_t a1 = byte_perm(r0[wd + 2], r1[wd + 2], sel);
                  const uint32_t a2 = byte_perm(r2[wd], r3[wd], sel);
                  const uint32_t a3 = byte_perm(r2[wd + 2], r3[wd + 2], sel);
                  const uint32_t lo[4] = {e4m3x2_to_f16x2(a0), e4m3x2_to_f16x2(a1), e4m3x2_to_f16x2(a2),
                                          e4m3x2_to_f16x2(a3)};
                  MOp::run(o[4 * wd + i], lo, pb0, pb1);
                  const uint32_t hi[4] = {e4m3x2_to_f16x2(a0 >> 16), e4m3x2_to_f16x2(a1 >> 16),
                                          e4m3x2_to_f16x2(a2 >> 16), e4m3x2_to_f16x2(a3 >> 16)};
                  MOp::run(o[4 * wd + i + 1], hi, pb0, pb1);
                }
              }
            }
          }
        } else {
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        if constexpr (!KV8) {
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
              const int key = wkey0 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
              const int d = kk * 16 + ((lane >> 3) & 1) * 8;
              const int c = (d & 63) >> 3;
              const uint32_t addr = kbase + (d >> 6) * Cfg::kPanelBytes + key * 128 + ((c ^ (key & 7)) << 4);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(addr, b0, b1, b2, b3);
              Op::run(s[2 * np], qf[kk], b0, b1);
              Op::run(s[2 * np + 1], qf[kk], b2, b3);
            }
          }
        } else {
          // e4m3 K rows are 128 bytes, 16-byte chunk c of key row r at (c ^ (r & 7)) * 16; in the permuted
          // k order a thread needs chunks 2tq and 2tq+1 of its key (r & 7 == gq): word kk holds the B
          // pairs of k step kk
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int key = wkey0 + nt * 8 + gq;
            const uint32_t rowa = kbase + key * 128;
            const uint4 c0 = lds_v4(rowa + (((2 * tq) ^ gq) << 4));
            const uint4 c1 = lds_v4(rowa + (((2 * tq + 1) ^ gq) << 4));
            const uint32_t kw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
              MOp::run(s[nt], qf[kk], e4m3x2_to_f16x2(kw[kk]), e4m3x2_to_f16x2(kw[kk] >> 16));
          }
        }
        // scale, mask, online softmax
        const bool need_mask = key0 + Cfg::kTile > P;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v = s[nt][e] * sl2r[e >> 1];
            if (need_mask) {
              const int key = key0 + wkey0 + nt * 8 + 2 * tq + (e & 1);
              const int h = e >> 1;
              bool vis = key < P || (key < L && ((mw[h] >> ((key - P) & 31)) & 1u));
              v = vis ? v : -INFINITY;
            }
            s[nt][e] = v;
          }
        }
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float mx = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float m_new = fmaxf(m_run[h], mx);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          alpha[h] = fast_exp2(m_run[h] - m_use);
          m_run[h] = m_new;
          float rs = 0.f;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float p0 = fast_exp2(s[nt][2 * h] - m_use);
            const float p1 = fast_exp2(s[nt][2 * h + 1] - m_use);
            s[nt][2 * h] = p0;
            s[nt][2 * h + 1] = p1;
            rs += p0 + p1;
          }
          l_run[h] = l_run[h] * alpha[h] + rs;
        }
        // O only needs rescaling when some row's running max moved (alpha is exactly 1 otherwise)
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
          for (int dt = 0; dt < DT; ++dt) {
            o[dt][0] *= alpha[0];
            o[dt][1] *= alpha[0];
            o[dt][2] *= alpha[1];
            o[dt][3] *= alpha[1];
          }
        }
        // O += P V
#pragma unroll
        for (int ks = 0; ks < KW / 16; ++ks) {
          uint32_t a[4];
          a[0] = MOp::pack(s[2 * ks][0], s[2 * ks][1]);
          a[1] = MOp::pack(s[2 * ks][2], s[2 * ks][3]);
          a[2] = MOp::pack(s[2 * ks + 1][0], s[2 * ks + 1][1]);
          a[3] = MOp::pack(s[2 * ks + 1][2], s[2 * ks + 1][3]);
          if constexpr (!KV8) {
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
              const int key = wkey0 + ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
              const int d = dp * 16 + (lane >> 4) * 8;
              const int c = (d & 63) >> 3;
              const uint32_t addr = vbase + (d >> 6) * Cfg::kPanelBytes + key * 128 + ((c ^ (key & 7)) << 4);
              uint32_t b0, b1, b2, b3;
              ldsm_x4_trans(addr, b0, b1, b2, b3);
              Op::run(o[2 * dp], a, b0, b1);
              Op::run(o[2 * dp + 1], a, b2, b3);
            }
          } else {
            // Output columns are permuted: column n of n tile dt is head dim n*16 + dt, so the B
            // fragments of a thread (column gq) are byte dt of chunk gq of key rows 2tq, 2tq+1, 2tq+8,
            // 2tq+9 (row & 7 == 2tq or 2tq+1), four 16-byte loads per 16 keys
            const int kr = wkey0 + ks * 16 + 2 * tq;
            const uint4 x0 = lds_v4(vbase + kr * 128 + ((gq ^ (2 * tq)) << 4));
            const uint4 x1 = lds_v4(vbase + (kr + 1) * 128 + ((gq ^ (2 * tq + 1)) << 4));
            const uint4 x2 = lds_v4(vbase + (kr + 8) * 128 + ((gq ^ (2 * tq)) << 4));
            const uint4 x3 = lds_v4(vbase + (kr + 9) * 128 + ((gq ^ (2 * tq + 1)) << 4));
            const uint32_t r0[4] = {x0.x, x0.y, x0.z, x0.w}, r1[4] = {x1.x, x1.y, x1.z, x1.w};
            const uint32_t r2[4] = {x2.x, x2.y, x2.z, x2.w}, r3[4] = {x3.x, x3.y, x3.z, x3.w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
              for (int i = 0; i < 4; i += 2) {
                // bytes (i of row 2tq, i of row 2tq+1, i+1 of row 2tq, i+1 of row 2tq+1)
                const uint32_t sel = i | ((4 + i) << 4) | ((i + 1) << 8) | ((5 + i) << 12);
                const uint32_t lo = byte_perm(r0[wd], r1[wd], sel);
                const uint32_t hi = byte_perm(r2[wd], r3[wd], sel);
                MOp::run(o[4 * wd + i], a, e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(hi));
                MOp::run(o[4 * wd + i + 1], a, e4m3x2_to_f16x2(lo >> 16), e4m3x2_to_f16x2(hi >> 16));
              }
            }
          }
        }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(empty_bar + stage));
      if (++stage == Cfg::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }

    // ---------------------------------------------------------------- segment epilogue
    // row sums: over the 4 lanes of a row, or (swapped form) over the 8 lanes of a query column
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if constexpr (SW) {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 4);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 8);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 16);
      } else {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
      }
    }
    if constexpr (KG > 1) {
      if constexpr (SW) {
        if (gq == 0) {
          m_pub[warp * 8 + 2 * tq] = m_run[0];
          m_pub[warp * 8 + 2 * tq + 1] = m_run[1];
        }
      } else if (tq == 0) {
        m_pub[warp * 16 + gq] = m_run[0];
        m_pub[warp * 16 + gq + 8] = m_run[1];
      }
      named_bar_sync(1, 128);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mstar = -INFINITY;
#pragma unroll
        for (int k2 = 0; k2 < KG; ++k2)
          mstar = fmaxf(mstar, SW ? m_pub[k2 * 8 + 2 * tq + h] : m_pub[(mt + k2 * MTS) * 16 + gq + 8 * h]);
        const float f = (m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - mstar);
        l_run[h] *= f;
#pragma unroll
        for (int dt = 0; dt < OT; ++dt) {
          if constexpr (SW) {   // elements h and 2 + h belong to query column 2tq + h
            o[dt][h] *= f;
            o[dt][2 + h] *= f;
          } else {
            o[dt][2 * h] *= f;
            o[dt][2 * h + 1] *= f;
          }
        }
        m_run[h] = mstar;
      }
      // deterministic sequential sum of the key groups' partial O through one scratch tile
      for (int mr = 0; mr < MTS; ++mr) {
        for (int kr = 0; kr < KG; ++kr) {
          if (mt == mr && kg == kr) {
            if (kr > 0) {
#pragma unroll
              for (int dt = 0; dt < OT; ++dt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[dt][e] += scratch[(dt * 4 + e) * 32 + lane];
              l_run[0] += scratch_l[lane];
              l_run[1] += scratch_l[32 + lane];
            }
            if (kr < KG - 1) {
#pragma unroll
              for (int dt = 0; dt < OT; ++dt)
#pragma unroll
                for (int e = 0; e < 4; ++e) scratch[(dt * 4 + e) * 32 + lane] = o[dt][e];
              scratch_l[lane] = l_run[0];
              scratch_l[32 + lane] = l_run[1];
            }
          }
          named_bar_sync(1, 128);
        }
      }
    }
    const bool owner = (kg == KG - 1);
    const bool whole_unit = (tbegin == 0 && tend == Tb);
    const int64_t unit_base = base_b + static_cast<int64_t>(j) * Tb;
    const int slot = 2 * static_cast<int>(blockIdx.x) + (first_segment ? 0 : 1);
    if (owner && SW) {
      // stage the normalised rows in shared memory ([8][D] floats, free once the key groups are summed),
      // then write them row by row with whole-row coalesced stores
      float* so = scratch;
      float inv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        inv[h] = (l_run[h] > 0.f ? 1.f / l_run[h] : 0.f) * vsc;
        if (gq == 0) scratch_l[2 * tq + h] = l_run[h] > 0.f ? m_run[h] + __log2f(l_run[h]) : -INFINITY;
      }
#pragma unroll
      for (int md = 0; md < OT; ++md) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // head dim of m row gq (e < 2) or gq + 8: md*16 + gq (+8), or gq*16 + md (+8) for e4m3 caches
          const int hd = KV8 ? gq * 16 + (e >> 1) * 8 + md : md * 16 + (e >> 1) * 8 + gq;
          so[(2 * tq + (e & 1)) * D + hd] = o[md][e] * inv[e & 1];
        }
      }
      __syncwarp();
      constexpr int PER = D / 32;   // values per lane and row
#pragma unroll 1
      for (int r = 0; r < ROWS; ++r) {
        const int R = rg * ROWS + r;
        const float* src = so + r * D + lane * PER;
        if (whole_unit) {
          if (R < p.G * p.C) {
            const bool valid = R < p.G * n;
            T* dst = static_cast<T*>(p.out) +
                     ((static_cast<int64_t>(b) * p.C + R / p.G) * p.Hq + g * p.G + R % p.G) * D + lane * PER;
            if constexpr (PER == 4) {
              uint2 x = make_uint2(0u, 0u);
              if (valid) {
                x.x = Op::pack(src[0], src[1]);
                x.y = Op::pack(src[2], src[3]);
              }
              *reinterpret_cast<uint2*>(dst) = x;
            } else {
              *reinterpret_cast<uint32_t*>(dst) = valid ? Op::pack(src[0], src[1]) : 0u;
            }
          }
        } else {
          float* dst = p.part_o + (static_cast<int64_t>(slot) * ROWS + r) * D + lane * PER;
          if constexpr (PER == 4)
            __stcg(reinterpret_cast<float4*>(dst), make_float4(src[0], src[1], src[2], src[3]));
          else
            __stcg(reinterpret_cast<float2*>(dst), make_float2(src[0], src[1]));
          if (lane == 0) __stcg(p.part_lse + static_cast<int64_t>(slot) * ROWS + r, scratch_l[r]);
        }
      }
      __syncwarp();
    } else if (owner) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int R = Rrow[h];
        const float inv = (l_run[h] > 0.f ? 1.f / l_run[h] : 0.f) * vsc;
        if (whole_unit) {
          if (R < p.G * p.C) {
            const int i = R / p.G, hh = R % p.G;
            T* dst = static_cast<T*>(p.out) + ((static_cast<int64_t>(b) * p.C + i) * p.Hq + g * p.G + hh) * D;
            if constexpr (!KV8) {
#pragma unroll
              for (int dt = 0; dt < DT; ++dt)
                *reinterpret_cast<uint32_t*>(dst + dt * 8 + 2 * tq) =
                    rvalid[h] ? Op::pack(o[dt][2 * h] * inv, o[dt][2 * h + 1] * inv) : 0u;
            } else {
              // permuted columns: this thread holds head dims tq*32 + j, j < 16 in o[j][2h], j >= 16 in
              // o[j - 16][2h + 1]
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int e = 2 * h + (v >> 1);
                const int d0 = (v & 1) * 8;
                uint4 x = make_uint4(0u, 0u, 0u, 0u);
                if (rvalid[h]) {
                  x.x = Op::pack(o[d0][e] * inv, o[d0 + 1][e] * inv);
                  x.y = Op::pack(o[d0 + 2][e] * inv, o[d0 + 3][e] * inv);
                  x.z = Op::pack(o[d0 + 4][e] * inv, o[d0 + 5][e] * inv);
                  x.w = Op::pack(o[d0 + 6][e] * inv, o[d0 + 7][e] * inv);
                }
                *reinterpret_cast<uint4*>(dst + tq * 32 + v * 8) = x;
              }
            }
          }
        } else {
          const int r = mt * 16 + gq + 8 * h;
          float* dst = p.part_o + (static_cast<int64_t>(slot) * ROWS + r) * D;
          if constexpr (!KV8) {
#pragma unroll
            for (int dt = 0; dt < DT; ++dt)
              __stcg(reinterpret_cast<float2*>(dst + dt * 8 + 2 * tq),
                     make_float2(o[dt][2 * h] * inv, o[dt][2 * h + 1] * inv));
          } else {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const int e = 2 * h + (v >> 2);
              const int d0 = (v & 3) * 4;
              __stcg(reinterpret_cast<float4*>(dst + tq * 32 + v * 4),
                     make_float4(o[d0][e] * inv, o[d0 + 1][e] * inv, o[d0 + 2][e] * inv, o[d0 + 3][e] * inv));
            }
          }
          if (tq == 0)
            __stcg(p.part_lse + static_cast<int64_t>(slot) * ROWS + r,
                   l_run[h] > 0.f ? m_run[h] + __log2f(l_run[h]) : -INFINITY);
        }
      }
    }
    if (!whole_unit && !p.defer_merge) {
      __threadfence();
      named_bar_sync(1, 128);
      const int u = (b * p.Hkv + g) * p.row_groups + rg;
      const UnitCtas uc = unit_ctas(p, unit_base, Tb, u, W, nC);
      const int c_first = uc.c_first, c_last = uc.c_last;
      if (tid == 0) {
        const uint32_t prev = atomicAdd(p.counters + u, 1u);
        const bool last = prev == static_cast<uint32_t>(c_last - c_first);
        if (last) {
          p.counters[u] = 0u;
          __threadfence();
        }
        sched->merge_flag = last ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (sched->merge_flag) {
        const int64_t row0 = static_cast<int64_t>(b) * p.C;
        merge_split_unit<T, D>(p, ROWS, ROWS, c_first, c_last, uc.first_odd, warp, lane,
                               [&](int r) -> MergeRow<T> {
                                 const int R = rg * ROWS + r;
                                 if (R >= p.G * p.C) return MergeRow<T>{nullptr, false};
                                 const int i = R / p.G;
                                 T* d = static_cast<T*>(p.out) + ((row0 + i) * p.Hq + g * p.G + R % p.G) * D;
                                 return MergeRow<T>{d, i < n};
                               });
      }
      named_bar_sync(1, 128);
    }

    // next unit
    first_segment = false;
    t += tend - tile;
    tile = 0;
    if (++j == HR) {
      j = 0;
      base_b += static_cast<int64_t>(Tb) * HR;
      if (++b < p.B) {
        L = clamp_context(p, b, false);
        Tb = tiles_of(L, Cfg::kTile);
      }
    }
  }
}

}  // namespace taco
