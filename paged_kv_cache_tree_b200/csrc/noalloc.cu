// paged_tree_attention_noalloc: the verify entry point for callers that must not allocate device
// memory.
//
// paged_tree_attention keeps a workspace for its split-KV partial results and grows it with
// cudaMalloc on first use. Some callers cannot allow that: code running under a fixed memory-pool
// budget (an inference server that reserves all free HBM for its KV cache up front), callers that
// must not trigger the implicit device synchronisation of cudaMalloc/cudaFree in the middle of a
// pipelined step, and hosts that forbid allocation after start-up. This variant computes the same
// result but takes its scratch (split-KV partials, arrival counters, error word) from a fixed array
// that lives in the library's device image instead of calling cudaMalloc.
//
// Kernel: the same choice as paged_tree_attention makes automatically. Wide packed tiles (G * C >= 48,
// G <= 128) run the tcgen05 kernel (one CTA per SM, 128-row partial slots); the others run the mma.sync
// kernel.
//
// Limits and rules:
//  - The scratch is kNoAllocScratchBytes = 24 MiB per device. Every GPU that loads the library holds
//    it until the process exits. It holds two partial slots per CTA of either kernel's full grid on a
//    148-SM B200 (the tcgen05 kernel's 128-row slots at head_dim 128 take 19.7 MB).
//  - At most kNoAllocMaxUnits = 65536 work units (batch * num_kv_heads * row groups). Larger calls are
//    rejected with TACO_ERR_UNSUPPORTED before anything is enqueued. The grid is capped so that the
//    partials fit in the scratch (on a GPU with more SMs than that, fewer CTAs than
//    paged_tree_attention uses).
//  - All calls on a device share the one array, and it keeps the previous call's contents. Each call
//    clears the arrival counters it needs on `stream` before its kernel runs. Two calls whose work
//    overlaps on the GPU (different streams without ordering between them) race on the scratch and
//    give wrong results: serialise them.
//  - The first call on a device (of this entry point or of taco_attn_check_noalloc) looks up the
//    array's device address with cudaGetSymbolAddress, with that device current; make that first call
//    before any stream capture begins.
//  - Device-side range violations (bad block ids, lengths) and wait timeouts are skipped as in
//    paged_tree_attention and recorded in this scratch's own error word. The word accumulates over
//    calls until taco_attn_check_noalloc reads and clears it (taco_attn_check_device does not see it).
//  - No cudaMalloc, cudaFree or other allocating call is made.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "device_common.cuh"
#include "launchers.h"
#include "taco_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(24) << 20;
constexpr int kNoAllocMaxUnits = 65536;
constexpr size_t kErrWordBytes = 256;
constexpr size_t kCounterBytes = size_t(kNoAllocMaxUnits) * 4;
constexpr size_t kPartialBytes = kNoAllocScratchBytes - kErrWordBytes - kCounterBytes;
constexpr int kMaxDevices = 64;

// The fixed scratch: [error word (256 B) | arrival counters (256 KiB) | partial lse | partial O].
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
unsigned char* g_scratch_addr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

// messages go to the same thread-local slot taco_attn_last_error() reads
taco_status fail(taco_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  taco::set_last_error_message(buf);
  return st;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device address of the scratch on the current device `dev`, looked up once per device (with `dev`
// current) and cached. Caller holds g_mu.
taco_status scratch_of(int dev, unsigned char** out) {
  if (!g_scratch_addr[dev]) {
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    e = cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = static_cast<unsigned char*>(addr);
  }
  *out = g_scratch_addr[dev];
  return TACO_OK;
}

}  // namespace

extern "C" taco_status paged_tree_attention_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* num_candidates, const uint32_t* tree_mask_bits, float scale,
    void* out, int32_t dtype, int32_t batch, int32_t max_candidates, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq, void* stream) {
  // same host-side checks as paged_tree_attention
  if (dtype != TACO_DTYPE_F16 && dtype != TACO_DTYPE_BF16) return fail(TACO_ERR_INVALID_ARG, "dtype must be F16 (0) or BF16 (1)");
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (max_candidates < 1) return fail(TACO_ERR_INVALID_ARG, "max_candidates must be >= 1");
  if (max_candidates > 32) return fail(TACO_ERR_UNSUPPORTED, "max_candidates must be <= 32");
  if (num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0)
    return fail(TACO_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
  if (head_dim != 64 && head_dim != 128) return fail(TACO_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (block_size < 8 || block_size > 256 || (block_size & (block_size - 1)) != 0)
    return fail(TACO_ERR_UNSUPPORTED, "block_size must be a power of two in [8, 256]");
  if (num_blocks < 1 || max_blocks_per_seq < 1) return fail(TACO_ERR_INVALID_ARG, "num_blocks and max_blocks_per_seq must be >= 1");
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size > INT32_MAX ||
      static_cast<int64_t>(max_blocks_per_seq) * block_size > INT32_MAX)
    return fail(TACO_ERR_UNSUPPORTED, "cache or block table too large for int32 indexing");
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !num_candidates || !tree_mask_bits || !out)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
        reinterpret_cast<uintptr_t>(out)) & 15u) != 0)
    return fail(TACO_ERR_INVALID_ARG, "q, k_cache, v_cache and out must be 16-byte aligned");
  if (!(scale == scale)) return fail(TACO_ERR_INVALID_ARG, "scale is NaN");
  if (batch == 0) return TACO_OK;

  const int G = num_q_heads / num_kv_heads;
  const int packed = G * max_candidates;
  const bool use_tc = packed >= 48 && G <= 128;  // as paged_tree_attention chooses for 16-bit caches
  const int cands_per_group = use_tc ? (max_candidates < 128 / G ? max_candidates : 128 / G) : 0;
  const int rows = use_tc ? 128 : taco::mma_rows_per_unit(packed);
  const int row_groups = use_tc ? (max_candidates + cands_per_group - 1) / cands_per_group : (packed + rows - 1) / rows;
  const int64_t units = static_cast<int64_t>(batch) * num_kv_heads * row_groups;
  if (units > kNoAllocMaxUnits)
    return fail(TACO_ERR_UNSUPPORTED,
                "paged_tree_attention_noalloc: %lld work units (batch * num_kv_heads * row groups) exceed the "
                "fixed scratch limit of %d; use paged_tree_attention",
                static_cast<long long>(units), kNoAllocMaxUnits);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  unsigned char* base = nullptr;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    taco_status st = scratch_of(dev, &base);  // one-time set-up on this device (the current one)
    if (st != TACO_OK) return st;
    sms = g_sm_count[dev];
  }

  // grid: the kernel's resident CTAs per SM, fewer if the partials (2 slots per CTA) would not fit
  const size_t slot_bytes = static_cast<size_t>(rows) * (head_dim + 1) * 4 + 512;
  const int max_grid = static_cast<int>(kPartialBytes / slot_bytes / 2);
  int grid = (use_tc ? 1 : taco::mma_ctas_per_sm(rows)) * sms;
  if (grid > max_grid) grid = max_grid;
  if (grid < 1) return fail(TACO_ERR_UNSUPPORTED, "scratch too small for one CTA");
  const size_t slots = 2 * static_cast<size_t>(grid);
  uint32_t* error_word = reinterpret_cast<uint32_t*>(base);
  uint32_t* counters = reinterpret_cast<uint32_t*>(base + kErrWordBytes);
  float* part_lse = reinterpret_cast<float*>(base + kErrWordBytes + kCounterBytes);
  float* part_o = reinterpret_cast<float*>(base + kErrWordBytes + kCounterBytes + round_up(slots * rows * 4, 256));

  // the counters of this call's units must start at zero; the error word keeps earlier calls' bits
  // until taco_attn_check_noalloc reads it
  e = cudaMemsetAsync(counters, 0, static_cast<size_t>(units) * 4, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaMemsetAsync(scratch): %s", cudaGetErrorString(e));

  // TMA descriptors of the two caches: rows of D elements, 64-column boxes of min(bs, tile keys) rows
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* sym = nullptr;
    cudaDriverEntryPointQueryResult qr{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &sym, 12000, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(sym);
  });
  if (!encode) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int tile = use_tc ? taco::tc_tile_keys() : taco::kTileKeys;
  const int rpc = block_size < tile ? block_size : tile;
  CUtensorMap maps[2];
  const void* caches[2] = {k_cache, v_cache};
  for (int m = 0; m < 2; ++m) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim),
                          static_cast<cuuint64_t>(num_blocks) * num_kv_heads * block_size};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(rpc)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&maps[m], dtype == TACO_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void*>(caches[m]), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  }
  // tcgen05 kernel: the query tile view [B*C, Hq, D], one box = 64 columns x G heads x the candidates of
  // one row group
  CUtensorMap qmap;
  if (use_tc) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                          static_cast<cuuint64_t>(batch) * max_candidates};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2, static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(cands_per_group)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&qmap, dtype == TACO_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", static_cast<int>(r));
  }

  taco::VerifyParams p{};
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.num_candidates = num_candidates;
  p.tree_mask_bits = tree_mask_bits;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.counters = counters;
  p.error_word = error_word;
  p.scale_log2 = scale * taco::kLog2e;
  p.B = batch;
  p.C = max_candidates;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = G;
  p.D = head_dim;
  p.bs = block_size;
  p.num_blocks = num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.rows_per_unit = rows;
  p.row_groups = row_groups;
  p.cands_per_group = cands_per_group;
  p.tile_keys = tile;
  p.l2_prefetch_tiles = use_tc ? taco::kTcPrefetchTiles : taco::kMmaPrefetchTiles;
  p.seg_cost = use_tc ? taco::tc_seg_cost(cands_per_group * G, false) : taco::mma_seg_cost(rows);
  e = use_tc ? taco::launch_verify_tc(maps[0], maps[1], qmap, p, dtype, grid, static_cast<cudaStream_t>(stream))
             : taco::launch_verify_mma(maps[0], maps[1], p, dtype, grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "verify kernel launch: %s", cudaGetErrorString(e));
  return TACO_OK;
}

// Reads and clears the scratch's error word (see the rules at the top of this file).
extern "C" taco_status taco_attn_check_noalloc(void* stream, uint32_t* bits_out) {
  if (bits_out) *bits_out = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  unsigned char* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    taco_status st = scratch_of(dev, &base);
    if (st != TACO_OK) return st;
  }
  uint32_t bits = 0;
  e = cudaMemcpy(&bits, base, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaMemcpy (noalloc error word): %s", cudaGetErrorString(e));
  if (bits_out) *bits_out = bits;
  if (bits == 0) return TACO_OK;
  e = cudaMemset(base, 0, 4);
  if (e != cudaSuccess) return fail(TACO_ERR_CUDA, "cudaMemset (noalloc error word): %s", cudaGetErrorString(e));
  return fail(TACO_ERR_DEVICE_CHECK, "paged_tree_attention_noalloc device check failed: bits 0x%x%s%s%s%s", bits,
              (bits & TACO_DEVERR_BLOCK_ID) ? " [block id out of range]" : "",
              (bits & TACO_DEVERR_CONTEXT_LEN) ? " [context length out of range]" : "",
              (bits & TACO_DEVERR_NUM_CAND) ? " [candidate count out of range]" : "",
              (bits & TACO_DEVERR_WAIT_TIMEOUT) ? " [pipeline wait timed out]" : "");
}
