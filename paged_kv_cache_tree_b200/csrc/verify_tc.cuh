// Verify kernel for wide packed query tiles (G * C >= 48 rows): the tcgen05 / tensor-memory path.
//
// The candidates of one (sequence, KV head) form up to 128 query rows (r = i_local * G + h'), the
// M = 128 operand of tcgen05.mma; this is how several candidates turn the decode GEMV into a GEMM
// ("大模型倍速推理引擎 TACO-LLM 的设计与实践", TurboAttention bullets under "整体方案分为两大部分").
// One CTA per SM, persistent over the same stream-K tile ranges as the mma.sync path, 128-key tiles:
//   warps 0, 10 producers: TMA loads of each segment's Q tile (3-D box over [B*C, Hq, D]) and of every
//               tile's K chunks (warp 0) and V chunks (warp 10) reached through the block table, into
//               separate K and V rings (K is released as soon as its Q K^T is done, V after its P V).
//               With e4m3 caches they load raw codes only, and the softmax warps widen each tile once
//               into the 16-bit layout;
//   warp 1      Q K^T issuer (one thread): S = Q K^T (M = 128, N = 128) into one of two tensor-memory
//               S buffers of 128 fp32 columns;
//   warp 11     P V issuer (one thread): O_w += P_w V_w per 64-key half w, with P read back from tensor
//               memory (A operand) and V from shared memory (MN-major B operand). Two issuing threads,
//               each waiting only for its own inputs in tile order, because issuing one tcgen05.mma or
//               commit costs a single thread tens of cycles and one thread doing both products plus the
//               polling between them became the bound of the whole kernel;
//   warps 2..9  two softmax warpgroups; warpgroup w takes keys [64 w, 64 w + 64) of every tile and owns
//               its own O accumulator in tensor memory. Thread r of a warpgroup owns query row r (lane
//               r): base-2 online softmax in fp32 whose reference max only moves when a row's max grows
//               by more than 2^8 (so O is rescaled rarely), P written back as 16-bit pairs into the S
//               buffer. At the end of a segment both warpgroups combine the two accumulators (each on
//               half of the head dims) and normalise, or write a split-KV partial.
// MMA completion is signalled with tcgen05.commit on mbarriers; every wait is bounded.
#pragma once

#include <type_traits>

#include "device_common.cuh"
#include "tc_ptx.cuh"

namespace taco {

// Keys per work tile of this kernel: Q K^T is one M = 128 x N = 128 product per k step. A
// tcgen05.mma with both operands in shared memory occupies the tensor core for about the same time
// at N = 64 as at N = 128 (measured on B200: about 120 cycles either way), so 64-key products spent
// half of the tensor core's time on nothing. Softmax warpgroup w takes keys [64 w, 64 w + 64) of
// every tile.
constexpr int kTcTileKeys = 128;

// KV8: e4m3 caches. Their tiles land in rings of raw codes and the eight softmax warps widen each one
// once (exactly) into a 16-bit stage of the same layout as a 16-bit cache's, so everything downstream
// is the 16-bit pipeline with f16 operands.
template <int D, bool KV8 = false>
struct TcCfg {
  static constexpr int kThreads = 384;
  static constexpr int kTK = kTcTileKeys;
  static constexpr int kHalf = kTK / 2;                    // keys per softmax warpgroup and tile
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = kTK * 128;            // kTK keys x 128 bytes
  static constexpr int kTensorBytes = kPanels * kPanelBytes;
  static constexpr int kKStages = KV8 ? ((D == 128) ? 2 : 4) : ((D == 128) ? 3 : 6);
  static constexpr int kVStages = kKStages;
  static constexpr int kRawStages = KV8 ? ((D == 128) ? 2 : 3) : 0;  // raw e4m3 tiles per tensor
  static constexpr int kRawBytes = kTK * D;                // one raw tile: kTK keys x D codes
  static constexpr int kQPanelBytes = 128 * 128;           // 128 rows x 128 bytes
  static constexpr int kQBytes = kPanels * kQPanelBytes;
  static constexpr int kSBufs = 2;                         // S/P buffers of kTK columns at 0, 128
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = 256;                        // O of warpgroup w at kOCol + w * 128
  static constexpr int kSharedBytes = 2048;
  static constexpr int kSmemBytes = 1024 + (kKStages + kVStages) * kTensorBytes + kQBytes +
                                    2 * kRawStages * kRawBytes + kSharedBytes;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct TcShared {
  // k_empty[s]: Q K^T of the tile in K stage s is done (its K slot is free; with as many K stages as
  // S buffers it also means the tile's S is ready). v_empty[s]: P V of the tile in V stage s is done
  // (its V slot and its S buffer are free, and its warpgroup's O holds it).
  // p_full[2 sb + w]: warpgroup w wrote its half of P into S buffer sb.
  uint64_t k_full[6], k_empty[6], v_full[6], v_empty[6];
  uint64_t q_full, q_empty, s_full[2], p_full[4], o_free;
  // e4m3 caches: raw tiles of K (index 0) and V (index 1) landed / widened by all eight softmax warps
  uint64_t raw_full[2][4], raw_empty[2][4];
  uint32_t tmem_base;
  int merge_flag, abort_flag;
  long long W, lo, hi, base_b;
  int nC, b;
  // per-row values the two softmax warpgroups exchange at a segment's end (reference max, then weighted sum);
  // the next segment's exchange comes after that segment's last P V, which waits for O to be
  // released, which both warpgroups do only after their reads here.
  float xs[2][128];
};

// 3-D TMA tile load (Q tile: x = column, y = head, z = sequence * C + candidate).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                            int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Split-KV partials of this kernel are stored transposed, [slot][head dim][128 rows] fp32, so that the
// 32 row-threads of a warp store and load one contiguous 128-byte line per instruction (a row-major
// layout made every warp instruction touch 32 lines, and the merge and epilogue ran at a fraction of
// L2's request rate).
//
// Combines the partials of one unit for row r, head dims [w D/2, (w + 1) D/2): one thread per
// (row, half), pieces s = 0 .. c_last - c_first in CTA order (slot of piece 0 is 2 c_first + 1 when it
// is not c_first's first segment, every other piece's is 2 c):
//   out = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),  M = max_s lse_s,
// pieces with lse = -inf (no visible key) weigh 0. The pieces' log-sum-exp and a 32-column chunk of
// two pieces are loaded together (unconditionally; a zero weight then selects 0); further pieces are
// folded in pairs with an online rescale.
template <typename T, int D>
__device__ __forceinline__ void merge_split_row_half(const VerifyParams& p, int r, int w, int c_first, int c_last,
                                                     bool first_odd, T* dst, bool active) {
  constexpr int H = D / 2;
  const int nsl = c_last - c_first + 1;
  auto slot_of = [&](int s) -> int64_t {
    const int c = c_first + s;
    return (s == 0 && first_odd) ? 2 * c + 1 : 2 * c;
  };
#pragma unroll 1
  for (int c0 = 0; c0 < H; c0 += 32) {
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.f;
    float M = -INFINITY, l = 0.f;
    for (int s0 = 0; s0 < nsl; s0 += 2) {
      float ls[2];
      float v[2][32];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool have = s0 + j < nsl;
        const int64_t sl = slot_of(have ? s0 + j : s0);
        ls[j] = __ldcg(p.part_lse + sl * 128 + r);
        const float* src = p.part_o + (sl * D + w * H + c0) * 128 + r;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[j][e] = __ldcg(src + e * 128);
        if (!have) ls[j] = -INFINITY;
      }
      const float mn = fmaxf(M, fmaxf(ls[0], ls[1]));
      if (mn == -INFINITY) continue;
      const float f = M == -INFINITY ? 0.f : exp2f(M - mn);
      float wt[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) wt[j] = ls[j] == -INFINITY ? 0.f : exp2f(ls[j] - mn);
      l = l * f + wt[0] + wt[1];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float t = acc[e] * f;
        if (wt[0] > 0.f) t = fmaf(wt[0], v[0][e], t);
        if (wt[1] > 0.f) t = fmaf(wt[1], v[1][e], t);
        acc[e] = t;
      }
      M = mn;
    }
    const float inv = (active && l > 0.f) ? 1.f / l : 0.f;
    uint32_t wv[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) wv[e] = active ? MmaOp<T>::pack(acc[2 * e] * inv, acc[2 * e + 1] * inv) : 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      *reinterpret_cast<uint4*>(dst + w * H + c0 + e * 8) = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
  }
}

template <typename T, int D, bool KV8>
__global__ void __launch_bounds__(384, 1)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ CUtensorMap tmap_q, const VerifyParams p) {
  using Cfg = TcCfg<D, KV8>;
  using Op = MmaOp<T>;                       // the output's type
  // operands of the tensor-core products: the queries' type, or f16 for e4m3 caches (codes widen
  // exactly to f16; the queries then come as f16 with a power-of-two scale per row)
  using POp = typename std::conditional<KV8, MmaOp<__half>, MmaOp<T>>::type;
  constexpr int SK = Cfg::kKStages;
  constexpr int SV = Cfg::kVStages;
  constexpr int NS = Cfg::kSBufs;
  constexpr int RS = Cfg::kRawStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value && !KV8;
  constexpr int TK = Cfg::kTK;
  constexpr int TH = Cfg::kHalf;
  constexpr uint32_t kIdescQK = tc::idesc_f16(kBf16 ? 1 : 0, 128, TK, 0);
  constexpr uint32_t kIdescPV = tc::idesc_f16(kBf16 ? 1 : 0, 128, D, 1);
  static_assert(sizeof(TcShared) <= Cfg::kSharedBytes, "shared bookkeeping too large");
  static_assert(!KV8 || SK == SV, "e4m3 widening indexes K and V stages alike");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kring = smem;
  uint8_t* vring = kring + SK * Cfg::kTensorBytes;
  uint8_t* qbuf = vring + SV * Cfg::kTensorBytes;
  uint8_t* rawring = qbuf + Cfg::kQBytes;  // e4m3: RS raw K tiles, then RS raw V tiles
  TcShared* sh = reinterpret_cast<TcShared*>(rawring + 2 * RS * Cfg::kRawBytes);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    // e4m3 caches: the eight softmax warps complete a stage (each widens sixteen rows of it) and free
    // a raw slot; 16-bit caches: the producer's TMA completes the stage
    constexpr uint32_t kFullArrivals = KV8 ? 8u : 1u;
    for (int s = 0; s < SK; ++s) {
      mbar_init(smem_addr(&sh->k_full[s]), kFullArrivals);
      mbar_init(smem_addr(&sh->k_empty[s]), 1);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(smem_addr(&sh->v_full[s]), kFullArrivals);
      mbar_init(smem_addr(&sh->v_empty[s]), 1);
    }
    mbar_init(smem_addr(&sh->q_full), 1);
    mbar_init(smem_addr(&sh->q_empty), 1);
    for (int j = 0; j < NS; ++j) mbar_init(smem_addr(&sh->s_full[j]), 1);
    for (int j = 0; j < 2 * NS; ++j) mbar_init(smem_addr(&sh->p_full[j]), 4);
    mbar_init(smem_addr(&sh->o_free), 8);
    for (int t = 0; t < 2; ++t)
      for (int s = 0; s < RS; ++s) {
        mbar_init(smem_addr(&sh->raw_full[t][s]), 1);
        mbar_init(smem_addr(&sh->raw_empty[t][s]), 8);
      }
    sh->merge_flag = 0;
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_addr(&sh->tmem_base), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  // inputs (and the cache an append just wrote) are read only after the grids this launch depends on;
  // after this library's own append (16-bit caches) only the producers wait, before the tiles that
  // hold its slots
  const bool late_wait = !KV8 && p.late_wait;
  if (!late_wait) grid_dependency_wait();
  if (warp == 0) {
    SchedStart s0 = schedule_start(p, blockIdx.x, gridDim.x);
    if (lane == 0) {
      sh->W = s0.W;
      sh->lo = s0.lo;
      sh->hi = s0.hi;
      sh->base_b = s0.base_b;
      sh->nC = s0.nC;
      sh->b = s0.b;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh->tmem_base;
  const int64_t W = sh->W;
  const int nC = sh->nC;
  if (static_cast<int>(blockIdx.x) >= nC) {
    if (warp == 1) tc::tmem_dealloc(tmem, Cfg::kTmemCols);
    return;
  }
  const int64_t lo = sh->lo, hi = sh->hi;
  volatile int* abort_flag = &sh->abort_flag;
  // barrier (and parity) that completes when S of tile k is in tensor memory
  constexpr bool kMergedS = (SK == NS);
  auto s_bar = [&](int64_t kk) -> uint32_t {
    return kMergedS ? smem_addr(&sh->k_empty[kk % SK]) : smem_addr(&sh->s_full[kk % NS]);
  };
  auto s_par = [&](int64_t kk) -> uint32_t { return static_cast<uint32_t>((kk / (kMergedS ? SK : NS)) & 1); };
  // barrier (and parity) that completes when P V of tile k is done
  auto pv_bar = [&](int64_t kk) -> uint32_t { return smem_addr(&sh->v_empty[kk % SV]); };
  auto pv_par = [&](int64_t kk) -> uint32_t { return static_cast<uint32_t>((kk / SV) & 1); };
  const int cpg = p.cands_per_group;
  const int qrows = cpg * p.G;

  if constexpr (KV8) {
    if (warp == 0 || warp == 10) {
      // -------------------------------------------------------------- e4m3 loaders
      // Warp 0 streams Q (f16, 3-D box) and K, warp 10 streams V: raw tiles of codes into a ring of
      // RS slots, in tile order, as far ahead as the slots allow. The eight softmax warps widen each
      // landed tile (sixteen rows each) into the 16-bit stage the tensor cores read and free the slot
      // (raw_empty counts their eight arrivals).
      const int t = (warp == 0) ? 0 : 1;
      const bool is_k = (t == 0);
      const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
      prefetch_tensormap(tmap);
      if (is_k) prefetch_tensormap(&tmap_q);
      const uint64_t policy = policy_evict_first();
      const int rpc = p.bs < TK ? p.bs : TK;
      const uint32_t chunk_bytes = static_cast<uint32_t>(rpc) * D;
      const uint32_t q_bytes = static_cast<uint32_t>(Cfg::kPanels * qrows * 128);
      uint8_t* raw = rawring + t * RS * Cfg::kRawBytes;
      TileLoadCursor lc;
      lc.init(p, sh->b, sh->base_b, lo, hi, is_k);
      bool ok = true;
      int q_issued_ui = -1;
      while (lc.have) {
        const bool seg_first = (lc.tl == lc.c.tile);
        const int ui = lc.c.ui;
        const int qb = lc.c.b, qj = lc.c.j;
        int row, nload;
        const bool mine = lc.chunk(p, TK, rpc, &row, &nload);
        const int rs = static_cast<int>(lc.k % RS);
        bool go = true;
        if (lane == 0) {
          // the slot's previous tile (RS tiles back) has been widened by all eight softmax warps
          go = ok && (*abort_flag == 0) &&
               (lc.k < RS ||
                mbar_wait(smem_addr(&sh->raw_empty[t][rs]), static_cast<uint32_t>(((lc.k / RS) - 1) & 1), p.error_word));
          if (!go) *abort_flag = 1;
          // armed on abort too (with no bytes), so that a widening warp never waits on it forever
          mbar_arrive_expect_tx(smem_addr(&sh->raw_full[t][rs]), go ? static_cast<uint32_t>(nload) * chunk_bytes : 0u);
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) ok = false;
        if (go && mine)
          tma_load_2d(smem_addr(raw + rs * Cfg::kRawBytes) + lane * chunk_bytes, tmap, smem_addr(&sh->raw_full[t][rs]),
                      0, row, policy);
        __syncwarp();
        if (is_k && seg_first && q_issued_ui < ui) {
          // the segment's Q tile, after its first raw K tile: the single Q buffer is free once the
          // previous segment's last Q K^T is done, which needs only tiles already loaded
          if (lane == 0) {
            bool gq = ok && (*abort_flag == 0) &&
                      mbar_wait(smem_addr(&sh->q_empty), static_cast<uint32_t>((ui & 1) ^ 1), p.error_word);
            if (!gq) *abort_flag = 1;
            mbar_arrive_expect_tx(smem_addr(&sh->q_full), gq ? q_bytes : 0u);
            if (gq) {
#pragma unroll
              for (int pn = 0; pn < Cfg::kPanels; ++pn)
                tma_load_3d(smem_addr(qbuf) + pn * Cfg::kQPanelBytes, &tmap_q, smem_addr(&sh->q_full), pn * 64,
                            (qj / p.row_groups) * p.G, qb * p.C + (qj % p.row_groups) * cpg);
            }
            if (!gq) ok = false;
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          q_issued_ui = ui;
        }
        lc.step(p);
      }
      // wait (bounded) for our own copies still landing: the last use of every raw slot, and the
      // last Q tile
      if (lane == 0) {
        for (int s = 0; s < RS; ++s) {
          const int64_t uses = lc.k / RS + (s < lc.k % RS ? 1 : 0);
          if (uses > 0)
            mbar_wait(smem_addr(&sh->raw_full[t][s]), static_cast<uint32_t>((uses - 1) & 1), p.error_word);
        }
        if (is_k && q_issued_ui >= 0)
          mbar_wait(smem_addr(&sh->q_full), static_cast<uint32_t>(q_issued_ui & 1), p.error_word);
      }
      if (!ok && lane == 0) *abort_flag = 1;
      return;
    }
  }
  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------------ producers
    // warp 0 streams Q and K, warp 10 streams V: both walk the same tiles and block table, so each
    // pays only its own share of the per-copy issue cost
    const bool is_k = (warp == 0);
    prefetch_tensormap(is_k ? &tmap_k : &tmap_v);
    if (is_k) prefetch_tensormap(&tmap_q);
    const uint64_t policy = policy_evict_first();
    const int rpc = p.bs < TK ? p.bs : TK;
    const int chunks_per_tile = TK / rpc;
    const uint32_t chunk_bytes = static_cast<uint32_t>(rpc) * 128u;
    const uint32_t q_bytes = static_cast<uint32_t>(Cfg::kPanels * qrows * 128);
    SegCursor cur;
    cur.init(p, sh->b, sh->base_b, lo, hi, true);
    int64_t k = 0;  // tile ordinal within the CTA
    // the V producer also asks L2 for both tensors of the tile pf_ahead tiles past its latest load
    const int pf_ahead = is_k ? 0 : p.l2_prefetch_tiles;
    TilePrefetcher<Cfg::kPanels, 64> pf;
    if (pf_ahead > 0) pf.init(p, sh->b, sh->base_b, lo, hi, SV);
    bool dep_done = !late_wait;
    while (cur.valid()) {
      const int g = cur.j / p.row_groups;
      const int rg = cur.j % p.row_groups;
      const int tend = cur.seg_end();
      const int L = cur.L;
      const int nblk = (L + p.bs - 1) / p.bs;
      const int32_t* bt_row = p.block_tables + static_cast<int64_t>(cur.b) * p.max_blocks;
      int win = -1000000;
      int32_t win_val = -1;
      // The segment's Q tile goes into the single Q buffer once the previous segment's last Q K^T
      // is done. K/V tiles of this segment may be issued first, but not more than SK - 1 of them:
      // from the SK-th on, a K slot's previous user belongs to this segment and needs its Q.
      bool q_issued = false;
      const int q_deadline = (tend - cur.tile - 1) < (SK - 2) ? (tend - cur.tile - 1) : (SK - 2);
      const uint32_t q_parity_prev = static_cast<uint32_t>((cur.ui & 1) ^ 1);
      for (int tl = cur.tile; tl < tend; ++tl, ++k) {
        if (!is_k) q_issued = true;
        if (!q_issued && lane == 0) {
          bool ready = (*abort_flag != 0) || mbar_test(smem_addr(&sh->q_empty), q_parity_prev);
          if (!ready && tl - cur.tile >= q_deadline) {
            ready = true;
            if (!mbar_wait(smem_addr(&sh->q_empty), q_parity_prev, p.error_word)) *abort_flag = 1;
          }
          if (ready) {
            const bool go = (*abort_flag == 0);
            mbar_arrive_expect_tx(smem_addr(&sh->q_full), go ? q_bytes : 0u);
            if (go) {
#pragma unroll
              for (int pn = 0; pn < Cfg::kPanels; ++pn)
                tma_load_3d(smem_addr(qbuf) + pn * Cfg::kQPanelBytes, &tmap_q, smem_addr(&sh->q_full), pn * 64,
                            g * p.G, cur.b * p.C + rg * cpg);
            }
            q_issued = true;
          }
        }
        q_issued = __shfl_sync(0xffffffffu, q_issued, 0);
        const int key0 = tl * TK;
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
          atomicOr(p.error_word, TACO_DEVERR_BLOCK_ID);
          ok = false;
        }
        const uint32_t bytes = __popc(__ballot_sync(0xffffffffu, ok)) * chunk_bytes * Cfg::kPanels;
        const int row = (blk * p.Hkv + g) * p.bs + (key0 + lane * rpc) % p.bs;
        if (!dep_done && key0 + TK > L - p.C) {  // the tile may hold slots the append wrote
          grid_dependency_wait();
          dep_done = true;
        }
        if (is_k) {  // K
          const int st = static_cast<int>(k % SK);
          bool go = true;
          if (lane == 0) {
            go = (*abort_flag == 0) &&
                 mbar_wait(smem_addr(&sh->k_empty[st]), static_cast<uint32_t>(((k / SK) & 1) ^ 1), p.error_word);
            if (!go) *abort_flag = 1;
            mbar_arrive_expect_tx(smem_addr(&sh->k_full[st]), go ? bytes : 0u);
          }
          go = __shfl_sync(0xffffffffu, go, 0);
          if (go && ok) {
            const uint32_t dst = smem_addr(kring + st * Cfg::kTensorBytes) + lane * chunk_bytes;
#pragma unroll
            for (int pn = 0; pn < Cfg::kPanels; ++pn)
              tma_load_2d(dst + pn * Cfg::kPanelBytes, &tmap_k, smem_addr(&sh->k_full[st]), pn * 64, row, policy);
          }
          __syncwarp();
        }
        if (!is_k) {  // V
          const int st = static_cast<int>(k % SV);
          bool go = true;
          if (lane == 0) {
            go = (*abort_flag == 0) &&
                 mbar_wait(smem_addr(&sh->v_empty[st]), static_cast<uint32_t>(((k / SV) & 1) ^ 1), p.error_word);
            if (!go) *abort_flag = 1;
            mbar_arrive_expect_tx(smem_addr(&sh->v_full[st]), go ? bytes : 0u);
          }
          go = __shfl_sync(0xffffffffu, go, 0);
          if (go && ok) {
            const uint32_t dst = smem_addr(vring + st * Cfg::kTensorBytes) + lane * chunk_bytes;
#pragma unroll
            for (int pn = 0; pn < Cfg::kPanels; ++pn)
              tma_load_2d(dst + pn * Cfg::kPanelBytes, &tmap_v, smem_addr(&sh->v_full[st]), pn * 64, row, policy);
          }
          __syncwarp();
          if (go && pf_ahead > 0) pf.prefetch(p, k + 1 + pf_ahead, &tmap_k, &tmap_v);
        }
      }
      cur.next_segment(p, true);
    }
    // wait (bounded) for our own copies: the last use of every ring slot and Q buffer
    if (lane == 0 && is_k) {
      for (int s = 0; s < SK; ++s) {
        const int64_t uses = k / SK + (s < k % SK ? 1 : 0);
        if (uses > 0) mbar_wait(smem_addr(&sh->k_full[s]), static_cast<uint32_t>((uses - 1) & 1), p.error_word);
      }
      if (cur.ui > 0) mbar_wait(smem_addr(&sh->q_full), static_cast<uint32_t>((cur.ui - 1) & 1), p.error_word);
    }
    if (lane == 0 && !is_k) {
      for (int s = 0; s < SV; ++s) {
        const int64_t uses = k / SV + (s < k % SV ? 1 : 0);
        if (uses > 0) mbar_wait(smem_addr(&sh->v_full[s]), static_cast<uint32_t>((uses - 1) & 1), p.error_word);
      }
    }
    return;
  }

  if (warp == 1 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuers
    // Warp 1 issues S = Q K^T, warp 11 issues O += P V, one thread each, tile by tile. Q K^T of tile
    // k needs its K landed, its S buffer (k % NS) free (P V of tile k - NS done) and, on a segment's
    // first tile, the segment's Q; P V of tile k needs its P written, its V landed and, on a
    // segment's first tile, O released by the previous segment's epilogue. Every wait is bounded;
    // a wait that gives up aborts the CTA and the issuer commits the rest of its barriers so that
    // nobody waits on it.
    if (lane == 0) {
      const bool is_qk = (warp == 1);
      TileWalker wk;
      wk.init(p, sh->b, sh->base_b, lo, hi);
      TileInfo ti;
      bool have = wk.next(p, ti);
      int64_t k = 0;
      // descriptor bases; every K step only adds a constant to the 14-bit start-address field
      const uint64_t q_desc = tc::smem_desc_sw128(smem_addr(qbuf), 16, 1024);
      const uint64_t k_desc = tc::smem_desc_sw128(smem_addr(kring), 16, 1024);
      const uint64_t v_desc = tc::smem_desc_sw128(smem_addr(vring), Cfg::kPanelBytes, 1024);
      bool ok = true;
      auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (*abort_flag != 0) return false;
        return mbar_wait(bar, parity, p.error_word);
      };
      if (is_qk) {
        for (; have; ++k, have = wk.next(p, ti)) {
          const int kst = static_cast<int>(k % SK);
          const int sb = static_cast<int>(k % NS);
          ok = wait(smem_addr(&sh->k_full[kst]), static_cast<uint32_t>((k / SK) & 1)) &&
               (k < NS || wait(pv_bar(k - NS), pv_par(k - NS))) &&
               (!ti.first || wait(smem_addr(&sh->q_full), static_cast<uint32_t>(ti.ui & 1)));
          if (!ok) break;
          tc::fence_after_sync();
          const uint64_t kd = k_desc + static_cast<uint64_t>((kst * Cfg::kTensorBytes) >> 4);
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(sb * TK);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            // panel (ks / 4), then 16 elements = 32 bytes along the 128-byte swizzled row
            const uint64_t qoff = static_cast<uint64_t>(((ks >> 2) * Cfg::kQPanelBytes + (ks & 3) * 32) >> 4);
            const uint64_t koff = static_cast<uint64_t>(((ks >> 2) * Cfg::kPanelBytes + (ks & 3) * 32) >> 4);
            tc::mma_ss(d_tmem, q_desc + qoff, kd + koff, kIdescQK, ks > 0 ? 1u : 0u);
          }
          if constexpr (!kMergedS) tc::commit(smem_addr(&sh->s_full[sb]));
          tc::commit(smem_addr(&sh->k_empty[kst]));
          if (ti.last) tc::commit(smem_addr(&sh->q_empty));
        }
      } else {
        for (; have; ++k, have = wk.next(p, ti)) {
          const int sb = static_cast<int>(k % NS);
          const int vs = static_cast<int>(k % SV);
          ok = wait(smem_addr(&sh->v_full[vs]), static_cast<uint32_t>((k / SV) & 1)) &&
               (!ti.first || ti.ui == 0 || wait(smem_addr(&sh->o_free), static_cast<uint32_t>((ti.ui - 1) & 1)));
          if (!ok) break;
          // each warpgroup's half as soon as its P is written: O_w += P_w V[64 w, 64 w + 64)
#pragma unroll 1
          for (int w = 0; w < 2; ++w) {
            ok = wait(smem_addr(&sh->p_full[2 * sb + w]), static_cast<uint32_t>((k / NS) & 1));
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t vd = v_desc + static_cast<uint64_t>((vs * Cfg::kTensorBytes + w * TH * 128) >> 4);
            const uint32_t a_tmem = tmem + static_cast<uint32_t>(sb * TK + w * TH);
            const uint32_t o_tmem = tmem + Cfg::kOCol + static_cast<uint32_t>(w * 128);
#pragma unroll
            for (int ks = 0; ks < TH / 16; ++ks) {
              // V as the MN-major B operand: 64-column panels kPanelBytes apart (LBO), 8-key groups
              // 1024 bytes apart (SBO); 16 keys per step = 2048 bytes; P: 16 keys = 8 packed columns
              tc::mma_ts(o_tmem, a_tmem + ks * 8, vd + static_cast<uint64_t>((ks * 2048) >> 4), kIdescPV,
                         (ti.first && ks == 0) ? 0u : 1u);
            }
          }
          if (!ok) break;
          tc::commit(smem_addr(&sh->v_empty[vs]));
        }
      }
      if (!ok) {
        // gave up (a wait ran out, or another role aborted): release everyone still waiting on us
        if (*abort_flag == 0) atomicOr(p.error_word, TACO_DEVERR_WAIT_TIMEOUT);
        *abort_flag = 1;
        for (; have; ++k, have = wk.next(p, ti)) {
          if (is_qk) {
            if constexpr (!kMergedS) tc::commit(smem_addr(&sh->s_full[k % NS]));
            tc::commit(smem_addr(&sh->k_empty[k % SK]));
            if (ti.last) tc::commit(smem_addr(&sh->q_empty));
          } else {
            tc::commit(smem_addr(&sh->v_empty[k % SV]));
          }
        }
      }
    }
    __syncwarp();
    tc::fence_before_sync();
    named_bar_sync(2, 320);
    if (warp == 1) {
      tc::fence_after_sync();
      tc::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    return;
  }

  // -------------------------------------------------------------------- softmax warpgroups
  const int wg = (warp - 2) >> 2;             // 0 or 1: owns the tiles with k % 2 == wg (warps 2..9)
  const int sub = warp & 3;                   // tensor-memory lane quarter of this warp
  const int r = sub * 32 + lane;              // query row owned by this thread
  const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
  const uint32_t my_o = tmem + lane_base + Cfg::kOCol + static_cast<uint32_t>(wg * 128);
  // e4m3 caches: softmax warp sw widens rows [16 sw, 16 sw + 16) of tile kk's raw K (t = 0) or V
  // (t = 1) codes into the tile's 16-bit stage, in the layout a 16-bit cache's TMA load leaves (two
  // 64-column 128-byte-swizzled panels at D = 128): cvt.rn.f16x2.e4m3x2 is exact, so the stage holds
  // exactly decode(code); the scales per KV head act on the scores and on O. Rows from zero_from on
  // (keys past the context) are written as zeros. The stage's previous tile must be done with it (its
  // Q K^T or P V complete; both needed only tiles widened earlier). Then this warp's arrival on the
  // stage's full barrier and on the raw slot's empty barrier (eight each); on abort too.
  auto widen = [&](int t, int64_t kk, int zero_from) {
    if constexpr (KV8) {
      const int sw = warp - 2;
      const int rs = static_cast<int>(kk % RS);
      const int cs = static_cast<int>(kk % SK);
      bool okw = (*abort_flag == 0);
      if (okw) okw = mbar_wait(smem_addr(&sh->raw_full[t][rs]), static_cast<uint32_t>((kk / RS) & 1), p.error_word);
      if (okw && kk >= SK)
        okw = mbar_wait(smem_addr(t == 0 ? &sh->k_empty[cs] : &sh->v_empty[cs]),
                        static_cast<uint32_t>(((kk / SK) - 1) & 1), p.error_word);
      if (!okw) *abort_flag = 1;
      if (okw) {
        const uint8_t* src = rawring + (t * RS + rs) * Cfg::kRawBytes;
        uint8_t* dst = (t == 0 ? kring : vring) + cs * Cfg::kTensorBytes;
        constexpr int CPR = D / 16;          // 16-code chunks per key row
        constexpr int PL = 16 * CPR / 32;    // chunks per lane (4 at D = 128, 2 at D = 64)
        uint4 v[PL];
#pragma unroll
        for (int j = 0; j < PL; ++j) {
          const int idx = j * 32 + lane;
          v[j] = lds_v4(smem_addr(src + (16 * sw + idx / CPR) * D + (idx % CPR) * 16));
        }
#pragma unroll
        for (int j = 0; j < PL; ++j) {
          const int idx = j * 32 + lane;
          const int row = 16 * sw + idx / CPR;
          const int c = idx % CPR;
          const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
          uint32_t h[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            h[2 * q] = e4m3x2_to_f16x2(w[q] & 0xffffu);
            h[2 * q + 1] = e4m3x2_to_f16x2(w[q] >> 16);
          }
          if (row >= zero_from) {
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = 0u;
          }
          // head dims [16c, 16c + 16) = 16-byte chunks 2(c % 4), 2(c % 4) + 1 of panel c / 4, swizzled
          uint8_t* prow = dst + (c >> 2) * Cfg::kPanelBytes + row * 128;
          const int j0 = 2 * (c & 3);
          *reinterpret_cast<uint4*>(prow + ((j0 ^ (row & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(prow + (((j0 + 1) ^ (row & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_addr(t == 0 ? &sh->k_full[cs] : &sh->v_full[cs]));
        mbar_arrive(smem_addr(&sh->raw_empty[t][rs]));
      }
    }
  };
  const int64_t n_tiles = hi - lo;  // this CTA's tiles, in the order every role walks them
  if constexpr (KV8) {
    if (n_tiles > 0) widen(0, 0, TK);
  }
  SegCursor cur;
  cur.init(p, sh->b, sh->base_b, lo, hi, false);
  int64_t k = 0;
  bool first_segment = true;
  // a segment's candidate count and this row's mask word, as loaded (the next segment's are loaded
  // at the start of the current one, so that a segment switch does not wait for them)
  // e4m3 caches: the row's logit scale also takes the KV head's K scale and the row's query scale
  auto load_seg_inputs = [&](int bb, int jj, int& n_raw, uint32_t& mw_raw, float& sl2) {
    n_raw = 0;
    mw_raw = 0u;
    sl2 = p.scale_log2;
    if (bb < p.B) {
      n_raw = __ldg(p.num_candidates + bb);
      const int gg = jj / p.row_groups;
      const int ii = (jj % p.row_groups) * cpg + r / p.G;
      if (r < qrows && ii < p.C) {
        mw_raw = __ldg(p.tree_mask_bits + static_cast<int64_t>(bb) * p.C + ii);
        if constexpr (KV8) {
          sl2 *= __ldg(p.k_scale + gg);
          if (p.q_scale != nullptr)
            sl2 *= __ldg(p.q_scale + (static_cast<int64_t>(bb) * p.C + ii) * p.Hq + gg * p.G + r % p.G);
        }
      }
    }
  };
  int n_raw_cur;
  uint32_t mw_raw_cur;
  float sl2_cur;
  load_seg_inputs(cur.b, cur.j, n_raw_cur, mw_raw_cur, sl2_cur);
  while (cur.valid()) {
    const int b = cur.b;
    const int g = cur.j / p.row_groups;
    const int rg = cur.j % p.row_groups;
    const int L = cur.L;
    const int tbegin = cur.tile;
    const int tend = cur.seg_end();
    const int Tb = cur.Tb;
    const int n = clamp_candidates_value(p, n_raw_cur, L, false);
    const int P = L - n;
    const uint32_t nmask = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
    const int i = rg * cpg + r / p.G;            // candidate of this row
    const int hh = r % p.G;
    const bool row_real = r < qrows && i < p.C;  // a row of the output
    const bool active = row_real && i < n;       // a row with a query
    const uint32_t mw = active ? (mw_raw_cur & nmask) : 0u;
    const float sl2 = sl2_cur;  // base-2 logit scale of this row
    const float vsc = KV8 ? __ldg(p.v_scale + g) : 1.f;
    {
      const bool same_b = cur.j + 1 < cur.HR;
      load_seg_inputs(same_b ? b : b + 1, same_b ? cur.j + 1 : 0, n_raw_cur, mw_raw_cur, sl2_cur);
    }

    float m_ref = -INFINITY;
    float l_run = 0.f;
    int64_t k_mine_last = -1;
    for (int tl = tbegin; tl < tend; ++tl, ++k) {
      const int key0 = tl * TK + wg * TH;   // this warpgroup's half of the tile
      const int sb = static_cast<int>(k % NS);
      if constexpr (KV8) {
        // the next tile's K (its Q K^T can then run during this tile's softmax), then this tile's V
        if (k + 1 < n_tiles) widen(0, k + 1, TK);
        widen(1, k, L - tl * TK);
      }
      const uint32_t s_col = tmem + lane_base + static_cast<uint32_t>(sb * TK + wg * TH);
      bool ok = (*abort_flag == 0);
      if (ok) ok = mbar_wait(s_bar(k), s_par(k), p.error_word);
      if (!ok) *abort_flag = 1;
      tc::fence_after_sync();
      uint32_t sraw[2][32];
      tc::ld_32x32b_x32(s_col, sraw[0]);
      tc::ld_32x32b_x32(s_col + 32, sraw[1]);
      tc::wait_ld();
      static_assert(TH == 64, "the softmax below holds one 64-column half tile per thread");
      // Row max of the raw scores (a positive scale_log2 commutes with max; otherwise the scaled
      // values are used). Masked keys become -inf; only the tiles that reach the candidates mask.
      const bool need_mask = key0 + TH > P;
      const bool pos_scale = sl2 > 0.f;
      float v[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = __uint_as_float(sraw[c >> 5][c & 31]);
      if (!pos_scale) {
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] *= sl2;
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = key0 + c;
          const bool vis = key < P || (key < L && ((mw >> ((key - P) & 31)) & 1u));
          v[c] = vis ? v[c] : -INFINITY;
        }
      }
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float a = tc::max3(v[8 * e], v[8 * e + 1], v[8 * e + 2]);
        a = tc::max3(a, v[8 * e + 3], v[8 * e + 4]);
        a = tc::max3(a, v[8 * e + 5], v[8 * e + 6]);
        m8[e] = fmaxf(a, v[8 * e + 7]);
      }
      const float mraw = tc::max3(tc::max3(m8[0], m8[1], m8[2]), tc::max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const bool first = (k_mine_last < 0);
      // rows without a query (padding) keep whatever their scores are; they never reach the output,
      // so they are simply kept out of the rescale decision
      float mx = pos_scale ? mraw * sl2 : mraw;  // row max of the base-2 logits
      if (!active) mx = first ? 0.f : m_ref;
      bool rescale = false;
      float alpha = 1.f;
      if (first) {
        m_ref = mx;
      } else if (mx > m_ref + 8.f) {
        rescale = true;
        alpha = fast_exp2(m_ref - mx);
        l_run *= alpha;
        m_ref = mx;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      // p = 2^(s * scale_log2 - m) on fp32 pairs; sums in four independent pair accumulators. The
      // fused form leaves every exponent off by the same t_ref - fl(t_ref) (t_ref the exact scaled
      // reference max), which cancels in the normalisation but reaches 2^(ulp(m) / 2): once a row's
      // reference max is 2^20 or more, the scores are scaled (rounded) first, so that the reference
      // key's exponent is exactly 0 (warp-uniform; ordinary logits never take this branch).
      bool scaled = !pos_scale;
      if (pos_scale && __any_sync(0xffffffffu, fabsf(m_use) >= 0x1p20f)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] *= sl2;
        scaled = true;
      }
      const float sc = scaled ? 1.f : sl2;
      const uint64_t sc2 = tc::f2(sc, sc);
      const uint64_t nm2 = tc::f2(-m_use, -m_use);
      uint64_t acc2[4] = {tc::f2(0.f, 0.f), tc::f2(0.f, 0.f), tc::f2(0.f, 0.f), tc::f2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float a0, a1;
        tc::f2_split(tc::f2_fma(tc::f2(v[2 * c], v[2 * c + 1]), sc2, nm2), a0, a1);
        const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
        acc2[c & 3] = tc::f2_add(acc2[c & 3], tc::f2(p0, p1));
        pk[c] = POp::pack(p0, p1);
      }
      {
        float s0, s1, s2, s3, s4, s5, s6, s7;
        tc::f2_split(acc2[0], s0, s1);
        tc::f2_split(acc2[1], s2, s3);
        tc::f2_split(acc2[2], s4, s5);
        tc::f2_split(acc2[3], s6, s7);
        l_run += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      }
      tc::st_32x32b_x32(s_col, pk);
      if (!KV8 && key0 + TH > L) {
        // keys >= L in this half: their V rows may be stale or NaN-poisoned; zero them once V has
        // landed (after P is written, so that the wait for V overlaps the softmax above; P V reads
        // them only after this warpgroup's p_full arrival below)
        const int vs = static_cast<int>(k % SV);
        bool okv = (*abort_flag == 0);
        if (okv) okv = mbar_wait(smem_addr(&sh->v_full[vs]), static_cast<uint32_t>((k / SV) & 1), p.error_word);
        if (!okv) *abort_flag = 1;
        int z0 = L - key0;
        if (z0 < 0) z0 = 0;
        uint8_t* vgen = vring + vs * Cfg::kTensorBytes;
        const int per_row = Cfg::kPanels * 8;
        for (int idx = r; idx < (TH - z0) * per_row; idx += 128) {
          const int row = wg * TH + z0 + idx / per_row;
          const int rem = idx % per_row;
          *reinterpret_cast<uint4*>(vgen + (rem / 8) * Cfg::kPanelBytes + row * 128 + (rem % 8) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // this warpgroup's O must be stable: the PV of its previous tile has to be complete
        const int64_t kprev = k_mine_last;
        bool okw = (*abort_flag == 0);
        if (okw)
          okw = mbar_wait(pv_bar(kprev), pv_par(kprev), p.error_word);
        if (!okw) *abort_flag = 1;
        tc::fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tc::ld_32x32b_x32(my_o + c * 32, o);
          tc::wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tc::st_32x32b_x32(my_o + c * 32, o);
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&sh->p_full[2 * sb + wg]));
      k_mine_last = k;
    }

    // ---------------------------------------------------------------- segment epilogue
    // Both warpgroups finish the segment together, each on half of the head dims of both O
    // accumulators: O = s_0 O_0 + s_1 O_1 with s_w = 2^(m_w - M) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)),
    // M = max(m_0, m_1) (m_w, l_w are warpgroup w's reference max and sum). The two exchange their
    // values through shared memory; this needs only the softmax state, so it runs while the segment's
    // last P V is still in flight.
    const bool have_keys = k_mine_last >= 0 && l_run > 0.f;
    // first the reference maxima, then each warpgroup's sum weighted by 2^(m_w - M): no log2(l) is ever
    // added to a max, which would lose it in rounding once |m| is large (logits of 2^20 and beyond)
    const float m_mine = have_keys ? m_ref : -INFINITY;
    sh->xs[wg][r] = m_mine;
    named_bar_sync(3, 256);
    const float m_other = sh->xs[wg ^ 1][r];
    const float Mx = fmaxf(m_mine, m_other);
    const float f_mine = m_mine == -INFINITY ? 0.f : fast_exp2(m_mine - Mx);
    const float f_other = m_other == -INFINITY ? 0.f : fast_exp2(m_other - Mx);
    named_bar_sync(3, 256);
    sh->xs[wg][r] = f_mine * (have_keys ? l_run : 0.f);
    named_bar_sync(3, 256);
    const float ltot = f_mine * (have_keys ? l_run : 0.f) + sh->xs[wg ^ 1][r];
    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
    const float LSE = ltot > 0.f ? Mx + __log2f(ltot) : -INFINITY;  // the segment's base-2 log-sum-exp
    const float s_mine = f_mine * inv, s_other = f_other * inv;
    const float s0r = wg == 0 ? s_mine : s_other;
    const float s1r = wg == 0 ? s_other : s_mine;
    const bool use0 = s0r > 0.f, use1 = s1r > 0.f;
    const float s0 = s0r * vsc;  // e4m3 caches: V's scale joins O here
    const float s1 = s1r * vsc;
    if (k_mine_last >= 0) {
      bool ok = (*abort_flag == 0);
      if (ok) ok = mbar_wait(pv_bar(k_mine_last), pv_par(k_mine_last), p.error_word);
      if (!ok) *abort_flag = 1;
    }
    tc::fence_after_sync();
    const bool whole_unit = (tbegin == 0 && tend == Tb);
    const int slot = 2 * static_cast<int>(blockIdx.x) + (first_segment ? 0 : 1);
    T* dst = static_cast<T*>(p.out) + ((static_cast<int64_t>(b) * p.C + i) * p.Hq + g * p.G + hh) * D;
    float* pdst = p.part_o + static_cast<int64_t>(slot) * D * 128 + r;  // transposed: [D][128] per slot
    const uint32_t o0 = tmem + lane_base + Cfg::kOCol;
    const uint32_t o1 = o0 + 128;
    // this warpgroup's D / 64 chunks of 32 head dims from both accumulators, loads issued together
    constexpr int NCH = D / 64;
    uint32_t oa[NCH][32], ob[NCH][32];
#pragma unroll
    for (int cc = 0; cc < NCH; ++cc) {
      tc::ld_32x32b_x32(o0 + (wg * NCH + cc) * 32, oa[cc]);
      tc::ld_32x32b_x32(o1 + (wg * NCH + cc) * 32, ob[cc]);
    }
    tc::wait_ld();
#pragma unroll
    for (int cc = 0; cc < NCH; ++cc) {
      const int c = wg * NCH + cc;
      const uint32_t(&a)[32] = oa[cc];
      const uint32_t(&bb)[32] = ob[cc];
      float x[32];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        x[e] = (use0 ? s0 * __uint_as_float(a[e]) : 0.f) + (use1 ? s1 * __uint_as_float(bb[e]) : 0.f);
      if (whole_unit) {
        if (row_real) {
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) wv[e] = active ? Op::pack(x[2 * e], x[2 * e + 1]) : 0u;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(dst + c * 32 + e * 8) =
                make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) __stcg(pdst + (c * 32 + e) * 128, x[e]);
      }
    }
    if (!whole_unit && wg == 0) __stcg(p.part_lse + static_cast<int64_t>(slot) * 128 + r, LSE);
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sh->o_free));

    if (!whole_unit && !p.defer_merge) {
      // the CTA that arrives last on the unit's counter combines every piece's partial
      __threadfence();
      named_bar_sync(1, 256);
      const int u = (b * p.Hkv + g) * p.row_groups + rg;
      const UnitCtas uc = unit_ctas(p, cur.unit_base(), Tb, u, W, nC);
      const int c_first = uc.c_first, c_last = uc.c_last;
      if (warp == 2 && lane == 0) {
        const uint32_t prev = atomicAdd(p.counters + u, 1u);
        const bool last = prev == static_cast<uint32_t>(c_last - c_first);
        if (last) {
          p.counters[u] = 0u;
          __threadfence();
        }
        sh->merge_flag = last ? 1 : 0;
      }
      named_bar_sync(1, 256);
      if (sh->merge_flag) {
        if (row_real) merge_split_row_half<T, D>(p, r, wg, c_first, c_last, uc.first_odd, dst, active);
      }
      named_bar_sync(1, 256);
    }
    first_segment = false;
    cur.next_segment(p, false);
  }
  tc::fence_before_sync();
  named_bar_sync(2, 320);
}

}  // namespace taco
