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
