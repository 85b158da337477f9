// Instantiations and launcher of the tcgen05 verify kernel.
#include "launchers.h"
#include "verify_tc.cuh"

namespace taco {

int tc_tile_keys() { return kTcTileKeys; }

int tc_smem_bytes(int D) { return D == 128 ? TcCfg<128>::kSmemBytes : TcCfg<64>::kSmemBytes; }

template <typename T, int D>
static cudaError_t launch_one(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                              const VerifyParams& p, int grid, cudaStream_t stream) {
  using Cfg = TcCfg<D>;
  auto kern = verify_tc_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(tk, tv, tq, p);
  return cudaGetLastError();
}

cudaError_t launch_verify_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const VerifyParams& p, int dtype, int grid, cudaStream_t stream) {
  if (dtype == TACO_DTYPE_BF16) {
    return p.D == 128 ? launch_one<__nv_bfloat16, 128>(tk, tv, tq, p, grid, stream)
                      : launch_one<__nv_bfloat16, 64>(tk, tv, tq, p, grid, stream);
  }
  return p.D == 128 ? launch_one<__half, 128>(tk, tv, tq, p, grid, stream)
                    : launch_one<__half, 64>(tk, tv, tq, p, grid, stream);
}

}  // namespace taco
