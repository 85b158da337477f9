// Instantiations and launcher of the mma.sync verify kernel.
#include "launchers.h"
#include "verify_mma.cuh"

namespace taco {

int mma_ctas_per_sm(int rows_per_unit) { return rows_per_unit == 8 ? MmaCfg<128, 0>::kCtasPerSm : MmaCfg<128, 1>::kCtasPerSm; }

int mma_rows_per_unit(int packed_rows) {
  if (packed_rows <= 8) return 8;     // swapped form
  if (packed_rows <= 16) return 16;
  if (packed_rows <= 32) return 32;
  return 64;
}

// (MT = rows / 16; 0 selects the swapped form for units of 8 rows)
int mma_tile_keys(int rows_per_unit, bool kv8) {
  const int mt = rows_per_unit / 16;
  if (!kv8) return MmaCfg<128, 1>::kTile;
  return mt == 0 ? MmaCfg<128, 0, true>::kTile : mt == 1 ? MmaCfg<128, 1, true>::kTile
         : mt == 2 ? MmaCfg<128, 2, true>::kTile : MmaCfg<128, 4, true>::kTile;
}

int mma_smem_bytes(int D, int rows_per_unit, bool kv8) {
  const int mt = rows_per_unit / 16;
  if (kv8)
    return mt == 0 ? MmaCfg<128, 0, true>::kSmemBytes : mt == 1 ? MmaCfg<128, 1, true>::kSmemBytes
           : mt == 2 ? MmaCfg<128, 2, true>::kSmemBytes : MmaCfg<128, 4, true>::kSmemBytes;
  if (D == 128) {
    return mt == 0 ? MmaCfg<128, 0>::kSmemBytes : mt == 1 ? MmaCfg<128, 1>::kSmemBytes
           : mt == 2 ? MmaCfg<128, 2>::kSmemBytes : MmaCfg<128, 4>::kSmemBytes;
  }
  return mt == 0 ? MmaCfg<64, 0>::kSmemBytes : mt == 1 ? MmaCfg<64, 1>::kSmemBytes
         : mt == 2 ? MmaCfg<64, 2>::kSmemBytes : MmaCfg<64, 4>::kSmemBytes;
}

template <typename T, int D, int MT, bool KV8 = false>
static cudaError_t launch_one(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p, int grid,
                              cudaStream_t stream) {
  using Cfg = MmaCfg<D, MT, KV8>;
  auto kern = verify_mma_kernel<T, D, MT, KV8>;
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
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_typed(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p, int grid,
                                cudaStream_t stream) {
  const int mt = p.rows_per_unit / 16;
  if (p.k_scale != nullptr) {  // e4m3 K/V (D = 128 only)
    if (mt == 0) return launch_one<T, 128, 0, true>(tk, tv, p, grid, stream);
    if (mt == 1) return launch_one<T, 128, 1, true>(tk, tv, p, grid, stream);
    if (mt == 2) return launch_one<T, 128, 2, true>(tk, tv, p, grid, stream);
    return launch_one<T, 128, 4, true>(tk, tv, p, grid, stream);
  }
  if (p.D == 128) {
    if (mt == 0) return launch_one<T, 128, 0>(tk, tv, p, grid, stream);
    if (mt == 1) return launch_one<T, 128, 1>(tk, tv, p, grid, stream);
    if (mt == 2) return launch_one<T, 128, 2>(tk, tv, p, grid, stream);
    return launch_one<T, 128, 4>(tk, tv, p, grid, stream);
  }
  if (mt == 0) return launch_one<T, 64, 0>(tk, tv, p, grid, stream);
  if (mt == 1) return launch_one<T, 64, 1>(tk, tv, p, grid, stream);
  if (mt == 2) return launch_one<T, 64, 2>(tk, tv, p, grid, stream);
  return launch_one<T, 64, 4>(tk, tv, p, grid, stream);
}

cudaError_t launch_verify_mma(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p, int dtype,
                              int grid, cudaStream_t stream) {
  if (dtype == TACO_DTYPE_BF16) return launch_typed<__nv_bfloat16>(tk, tv, p, grid, stream);
  return launch_typed<__half>(tk, tv, p, grid, stream);
}

}  // namespace taco
