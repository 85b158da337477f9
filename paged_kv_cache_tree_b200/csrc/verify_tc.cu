// Instantiations and launcher of the tcgen05 verify kernel.
#include "launchers.h"
#include "verify_tc.cuh"

namespace taco {

int tc_tile_keys() { return kTcTileKeys; }

int tc_smem_bytes(int D, bool kv8) {
  if (kv8) return D == 128 ? TcCfg<128, true>::kSmemBytes : TcCfg<64, true>::kSmemBytes;
  return D == 128 ? TcCfg<128>::kSmemBytes : TcCfg<64>::kSmemBytes;
}

template <typename T, int D, bool KV8>
static cudaError_t launch_one(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                              const VerifyParams& p, int grid, cudaStream_t stream) {
  using Cfg = TcCfg<D, KV8>;
  auto kern = verify_tc_kernel<T, D, KV8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // programmatic stream serialization: the prologue may overlap the previous kernel's tail; the
  // kernel waits for it (griddepcontrol.wait) before touching any input
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, bool KV8>
static cudaError_t launch_typed(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                                const VerifyParams& p, int grid, cudaStream_t stream) {
  return p.D == 128 ? launch_one<T, 128, KV8>(tk, tv, tq, p, grid, stream)
                    : launch_one<T, 64, KV8>(tk, tv, tq, p, grid, stream);
}

cudaError_t launch_verify_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const VerifyParams& p, int dtype, int grid, cudaStream_t stream) {
  const bool kv8 = p.k_scale != nullptr;
  if (dtype == TACO_DTYPE_BF16)
    return kv8 ? launch_typed<__nv_bfloat16, true>(tk, tv, tq, p, grid, stream)
               : launch_typed<__nv_bfloat16, false>(tk, tv, tq, p, grid, stream);
  return kv8 ? launch_typed<__half, true>(tk, tv, tq, p, grid, stream)
             : launch_typed<__half, false>(tk, tv, tq, p, grid, stream);
}

// ------------------------------------------------------------------------------------------------
// bf16 queries for e4m3 caches on the tcgen05 path: the tensor cores take f16 x f16 there (e4m3 codes
// widen exactly to f16), so each query row is multiplied by the power of two 2^k that puts its largest
// magnitude in [2^14, 2^15) and rounded to f16 (exact for every element down to 2^-29 of the row's
// largest); 2^-k is stored per row and joins the row's logit scale. One warp per row.
__global__ void __launch_bounds__(256) q_to_f16_kernel(const __nv_bfloat16* __restrict__ q, __half* __restrict__ q16,
                                                       float* __restrict__ qscale, int64_t rows, int D) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int per = D / 32;  // 2 or 4 values per lane
  const __nv_bfloat16* src = q + row * D + lane * per;
  float x[4];
  float mx = 0.f;
  for (int e = 0; e < per; ++e) {
    x[e] = __bfloat162float(src[e]);
    mx = fmaxf(mx, fabsf(x[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  int k = 0;
  if (mx > 0.f && mx <= FLT_MAX) {
    const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;
    k = 14 - e < 64 ? 14 - e : 64;
  }
  // 2^k and 2^-k as float bit patterns (k in [-113, 64] keeps both normal)
  const float up = __uint_as_float(static_cast<uint32_t>(127 + k) << 23);
  __half* dst = q16 + row * D + lane * per;
  for (int e = 0; e < per; ++e) dst[e] = __float2half_rn(x[e] * up);
  if (lane == 0) qscale[row] = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
}

cudaError_t launch_q_to_f16(const void* q, void* q16, float* qscale, int64_t rows, int D, cudaStream_t stream) {
  const int64_t threads = rows * 32;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  q_to_f16_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), static_cast<__half*>(q16), qscale,
                                              rows, D);
  return cudaGetLastError();
}

}  // namespace taco
