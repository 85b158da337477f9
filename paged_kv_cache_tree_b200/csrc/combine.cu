// The log-sum-exp combine of split-KV partials as a kernel of its own (step A9): after a verify launch
// whose split units only wrote their partials, every split unit's output rows are merged here.
//
// The pages decouple the on-chip resources from the sequence length for long sequences
// ("大模型倍速推理引擎 TACO-LLM 的设计与实践", TurboAttention bullets under "整体方案分为两大部分"): a
// long unit is cut into pieces that different CTAs attend, and their results are combined. For units cut
// into many pieces (few units against many CTAs, e.g. a handful of 128 k-token sequences), the merge by
// the last CTA to finish a unit is a serial tail at the end of the verify launch. This kernel instead
// gives every (unit, output row) its own warp, so all merges run at once and each is two round trips.
//
// It recomputes the verify's weighted work split from the same parameters to find each unit's pieces
// (unit_ctas). Partials come in either verify kernel's layout: the mma.sync kernel's O [slot][row][D]
// (a warp per output row, lanes along the head dims) or the tcgen05 kernel's transposed O [slot][D][128]
// (a warp per 32 rows x 32 head dims, lanes along the rows); lse [slot][row] in base 2, O normalised.
// For every element the pieces are summed in CTA order, so the result does not depend on timing.
#include "device_common.cuh"
#include "launchers.h"

namespace taco {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 8;  // pieces whose loads are in flight together

// Unit u's place in the weighted split, as the verify computed it: whether it was split, and its pieces.
__device__ __forceinline__ UnitCtas unit_place(const VerifyParams& p, int u, int grid, int& L) {
  const int HR = p.Hkv * p.row_groups;
  const int b = u / HR, j = u % HR;
  const int lane = threadIdx.x & 31;
  int64_t Wr = 0, base_b = 0;
  for (int bb = lane; bb < p.B; bb += 32) {
    const int64_t t = static_cast<int64_t>(tiles_of(clamp_context(p, bb, false), p.tile_keys)) * HR;
    Wr += t;
    if (bb < b) base_b += t;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Wr += __shfl_xor_sync(0xffffffffu, Wr, o);
    base_b += __shfl_xor_sync(0xffffffffu, base_b, o);
  }
  L = clamp_context(p, b, false);
  const int Tb = tiles_of(L, p.tile_keys);
  const int64_t W = Wr + static_cast<int64_t>(p.seg_cost) * p.B * HR;
  const int nC = static_cast<int>(Wr < grid ? Wr : grid);
  return unit_ctas(p, base_b + static_cast<int64_t>(j) * Tb, Tb, u, W, nC);
}

template <typename T, int D>
__global__ void __launch_bounds__(kCombineThreads) combine_split_kernel(const VerifyParams p, int grid) {
  grid_dependency_wait();  // the verify's partials are complete and visible
  const int HR = p.Hkv * p.row_groups;
  const int units = p.B * HR;
  const int ROWS = p.rows_per_unit;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(units) * ROWS) return;
  const int u = static_cast<int>(wid / ROWS), r = static_cast<int>(wid % ROWS);
  const int b = u / HR, j = u % HR;
  int L;
  const UnitCtas uc = unit_place(p, u, grid, L);
  if (uc.c_first == uc.c_last) return;  // a whole unit: the verify wrote its rows
  const int g = j / p.row_groups, rg = j % p.row_groups;
  const int R = rg * ROWS + r;
  if (R >= p.G * p.C) return;  // a padding row of the unit's tile: no output row
  const int i = R / p.G;
  const int n = clamp_candidates(p, b, L, false);
  T* dst = static_cast<T*>(p.out) + ((static_cast<int64_t>(b) * p.C + i) * p.Hq + g * p.G + R % p.G) * D;
  const int nsl = uc.c_last - uc.c_first + 1;
  auto slot_of = [&](int s) -> int64_t {
    const int c = uc.c_first + s;
    return (s == 0 && uc.first_odd) ? 2 * c + 1 : 2 * c;
  };
  // the pieces' largest lse, then every piece weighted by 2^(lse - M)
  float M = -INFINITY;
  for (int s = lane; s < nsl; s += 32) M = fmaxf(M, __ldcg(p.part_lse + slot_of(s) * ROWS + r));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  constexpr int V = D / 32;
  static_assert(V == 2 || V == 4, "head_dim 64 or 128");
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  float l = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < nsl; s0 += kCombineBatch) {
      float ls[kCombineBatch], v[kCombineBatch][V];
#pragma unroll
      for (int k = 0; k < kCombineBatch; ++k) {
        const int s = s0 + k;
        ls[k] = -INFINITY;
#pragma unroll
        for (int e = 0; e < V; ++e) v[k][e] = 0.f;
        if (s < nsl) {
          const int64_t sl = slot_of(s);
          ls[k] = __ldcg(p.part_lse + sl * ROWS + r);
          const float* src = p.part_o + (sl * ROWS + r) * D + lane * V;
          if constexpr (V == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(src));
            v[k][0] = x.x;
            v[k][1] = x.y;
            v[k][2] = x.z;
            v[k][3] = x.w;
          } else {
            const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
            v[k][0] = x.x;
            v[k][1] = x.y;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kCombineBatch; ++k) {
        if (ls[k] == -INFINITY) continue;  // the piece saw no visible key
        const float w = exp2f(ls[k] - M);
        l += w;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = fmaf(w, v[k][e], acc[e]);
      }
    }
  }
  const bool active = i < n;
  const float inv = (active && l > 0.f) ? 1.f / l : 0.f;
  uint32_t w2[V / 2];
#pragma unroll
  for (int e = 0; e < V / 2; ++e) w2[e] = active ? MmaOp<T>::pack(acc[2 * e] * inv, acc[2 * e + 1] * inv) : 0u;
  if constexpr (V == 4)
    *reinterpret_cast<uint2*>(dst + lane * V) = make_uint2(w2[0], w2[1]);
  else
    *reinterpret_cast<uint32_t*>(dst + lane * V) = w2[0];
}

// tcgen05 partials [slot][D][128 rows]: warp (unit, 32-row block, 32-column block), lane = row
template <typename T, int D>
__global__ void __launch_bounds__(kCombineThreads) combine_split_transposed_kernel(const VerifyParams p, int grid) {
  grid_dependency_wait();
  constexpr int CB = D / 32;  // column blocks
  const int HR = p.Hkv * p.row_groups;
  const int units = p.B * HR;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(units) * 4 * CB) return;
  const int u = static_cast<int>(wid / (4 * CB));
  const int rb = static_cast<int>(wid % (4 * CB)) / CB, cb = static_cast<int>(wid % CB);
  int L;
  const UnitCtas uc = unit_place(p, u, grid, L);
  if (uc.c_first == uc.c_last) return;  // a whole unit: the verify wrote its rows
  const int b = u / HR, j = u % HR;
  const int g = j / p.row_groups, rg = j % p.row_groups;
  const int r = rb * 32 + lane;
  const int i = rg * p.cands_per_group + r / p.G;
  if (r >= p.cands_per_group * p.G || i >= p.C) return;  // not a row of the output (no warp-wide step follows)
  const int n = clamp_candidates(p, b, L, false);
  const int nsl = uc.c_last - uc.c_first + 1;
  auto slot_of = [&](int s) -> int64_t {
    const int c = uc.c_first + s;
    return (s == 0 && uc.first_odd) ? 2 * c + 1 : 2 * c;
  };
  float M = -INFINITY;
  for (int s = 0; s < nsl; ++s) M = fmaxf(M, __ldcg(p.part_lse + slot_of(s) * 128 + r));
  float acc[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) acc[c] = 0.f;
  float l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsl; ++s) {
      const int64_t sl = slot_of(s);
      const float ls = __ldcg(p.part_lse + sl * 128 + r);
      if (ls == -INFINITY) continue;
      const float w = exp2f(ls - M);
      l += w;
      const float* src = p.part_o + (sl * D + cb * 32) * 128 + r;
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = __ldcg(src + c * 128);
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = fmaf(w, v[c], acc[c]);
    }
  }
  const bool active = i < n;
  const float inv = (active && l > 0.f) ? 1.f / l : 0.f;
  T* dst = static_cast<T*>(p.out) + ((static_cast<int64_t>(b) * p.C + i) * p.Hq + g * p.G + r % p.G) * D + cb * 32;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w4[e] = active ? MmaOp<T>::pack(acc[q * 8 + 2 * e] * inv, acc[q * 8 + 2 * e + 1] * inv) : 0u;
    reinterpret_cast<uint4*>(dst)[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

template <typename T, int D, bool kTransposed>
cudaError_t launch_t(const VerifyParams& p, int grid, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.Hkv * p.row_groups * (kTransposed ? 4 * (D / 32) : p.rows_per_unit);
  const int64_t blocks = (warps * 32 + kCombineThreads - 1) / kCombineThreads;
  // programmatic stream serialization: the CTAs may be placed while the verify's last CTAs finish;
  // each waits (griddepcontrol.wait) for the whole verify before reading a partial
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (kTransposed) return cudaLaunchKernelEx(&cfg, combine_split_transposed_kernel<T, D>, p, grid);
  return cudaLaunchKernelEx(&cfg, combine_split_kernel<T, D>, p, grid);
}

}  // namespace

cudaError_t launch_combine_split(const VerifyParams& p, int dtype, int grid, bool transposed, cudaStream_t stream) {
  const bool bf = dtype == TACO_DTYPE_BF16, d128 = p.D == 128;
  if (transposed) {
    if (bf) return d128 ? launch_t<__nv_bfloat16, 128, true>(p, grid, stream) : launch_t<__nv_bfloat16, 64, true>(p, grid, stream);
    return d128 ? launch_t<__half, 128, true>(p, grid, stream) : launch_t<__half, 64, true>(p, grid, stream);
  }
  if (bf) return d128 ? launch_t<__nv_bfloat16, 128, false>(p, grid, stream) : launch_t<__nv_bfloat16, 64, false>(p, grid, stream);
  return d128 ? launch_t<__half, 128, false>(p, grid, stream) : launch_t<__half, 64, false>(p, grid, stream);
}

}  // namespace taco
