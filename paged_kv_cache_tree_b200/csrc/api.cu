// Host side of libtaco_attn: argument validation, per-device workspace, TMA descriptors and
// kernel dispatch behind the C ABI declared in taco_attn.h.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "device_common.cuh"
#include "launchers.h"
#include "taco_attn.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAbiVersion = 8;

thread_local std::string g_last_error;

taco_status fail(taco_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

taco_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TACO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Workspace of one (device, stream): [error word | counters | partial lse | partial O]. Calls on
// different streams never share one, so they may overlap on the GPU.
struct Workspace {
  uint8_t* base = nullptr;
  size_t bytes = 0;
  uint32_t* error_word = nullptr;
  uint32_t* counters = nullptr;
  size_t counters_cap = 0;
  float* part_lse = nullptr;
  size_t lse_cap = 0;  // floats
  float* part_o = nullptr;
  size_t o_cap = 0;    // floats
  uint8_t* qbuf = nullptr;  // e4m3 tcgen05 path: f16 query rows, then one float scale per row
  size_t q_cap = 0;         // bytes
};

std::mutex g_mu;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;  // keyed by (device, stream handle)
int g_sm_count[kMaxDevices];
int64_t g_opt_grid = 0;
int64_t g_opt_kernel = 0;
int64_t g_opt_prefetch = -1;  // -1 = the kernel's default distance
int64_t g_opt_stall = 0;      // test knob: 0 = off, t + 1 = CTA 0 leaves tile t unarmed (mma.sync kernel)
int64_t g_opt_seg_cost = -1;  // -1 = the kernel's default segment cost of the work split
int64_t g_opt_combine = 0;    // 0 = automatic, 1 = merge inside the verify, 2 = separate combine kernel
// kernels the calling thread's last attention call enqueued
thread_local int g_last_launches = 0;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// SM count of device `dev`. Caller holds g_mu.
taco_status sm_count_of(int dev, int* out) {
  if (g_sm_count[dev] == 0) {
    cudaError_t e = cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  *out = g_sm_count[dev];
  return TACO_OK;
}

// Make sure the workspace of (device `dev`, `stream`) has room and return it in *out; returns a status.
// Caller holds g_mu.
taco_status ensure_workspace(int dev, void* stream, size_t counters, size_t lse_floats, size_t o_floats,
                             Workspace** out, size_t q_bytes = 0) {
  Workspace& w = g_ws[std::make_pair(dev, reinterpret_cast<uintptr_t>(stream))];
  *out = &w;
  if (w.base && counters <= w.counters_cap && lse_floats <= w.lse_cap && o_floats <= w.o_cap && q_bytes <= w.q_cap)
    return TACO_OK;
  // grow (keeping at least the old capacities); the old buffer may still be in use by queued
  // work, so wait for the device before freeing it
  counters = std::max(counters, w.counters_cap);
  lse_floats = std::max(lse_floats, w.lse_cap);
  o_floats = std::max(o_floats, w.o_cap);
  q_bytes = std::max(q_bytes, w.q_cap);
  const size_t off_counters = 256;
  const size_t off_lse = off_counters + round_up(counters * 4, 256);
  const size_t off_o = off_lse + round_up(lse_floats * 4, 256);
  const size_t off_q = off_o + round_up(o_floats * 4, 256);
  const size_t total = off_q + round_up(q_bytes, 256);
  uint32_t old_err = 0;
  if (w.base) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize (workspace grow)");
    cudaMemcpy(&old_err, w.error_word, 4, cudaMemcpyDeviceToHost);
    cudaFree(w.base);
    w = Workspace{};
  }
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, total);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc (workspace)");
  e = cudaMemset(p, 0, off_lse);  // error word and counters start at zero
  if (e != cudaSuccess) {
    cudaFree(p);
    return cuda_fail(e, "cudaMemset (workspace)");
  }
  if (old_err) cudaMemcpy(p, &old_err, 4, cudaMemcpyHostToDevice);
  w.base = static_cast<uint8_t*>(p);
  w.bytes = total;
  w.error_word = reinterpret_cast<uint32_t*>(w.base);
  w.counters = reinterpret_cast<uint32_t*>(w.base + off_counters);
  w.counters_cap = counters;
  w.part_lse = reinterpret_cast<float*>(w.base + off_lse);
  w.lse_cap = lse_floats;
  w.part_o = reinterpret_cast<float*>(w.base + off_o);
  w.o_cap = o_floats;
  w.qbuf = w.base + off_q;
  w.q_cap = q_bytes;
  return TACO_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* sym = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &sym, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(sym);
  });
  return fn;
}

// [NB * Hkv * bs rows, D columns] view of a cache; box = one 128-byte swizzle row (64 16-bit values,
// or 128 e4m3 codes when kv8) x rows_per_chunk rows.
// raw_rows (e4m3 only): whole D-byte rows, no swizzle (the tcgen05 path widens them in shared memory).
taco_status make_cache_map(CUtensorMap* map, const void* base, int dtype, int D, int64_t rows, int rows_per_chunk,
                           bool kv8 = false, bool raw_rows = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int elt = kv8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * elt};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(raw_rows ? D : 128 / elt), static_cast<cuuint32_t>(rows_per_chunk)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType ty = kv8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                     : (dtype == TACO_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  CUresult r = enc(map, ty, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   raw_rows ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TACO_OK;
}

// Query tile view [B*C, Hq, D]; box = 64 columns x G heads x cands_per_group candidates, so one box
// holds the packed rows r = i * G + h' of one (sequence, KV head, row group).
taco_status make_query_map(CUtensorMap* map, const void* q, int dtype, int D, int Hq, int64_t bc, int G,
                           int cands_per_group) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(bc)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(cands_per_group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype == TACO_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TACO_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", static_cast<int>(r));
  return TACO_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

taco_status check_common(int32_t dtype, int32_t batch, int32_t max_candidates, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t max_blocks) {
  if (dtype != TACO_DTYPE_F16 && dtype != TACO_DTYPE_BF16) return fail(TACO_ERR_INVALID_ARG, "dtype must be F16 (0) or BF16 (1)");
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (max_candidates < 1) return fail(TACO_ERR_INVALID_ARG, "max_candidates must be >= 1");
  if (max_candidates > 32) return fail(TACO_ERR_UNSUPPORTED, "max_candidates must be <= 32 (one 32-bit mask word per row)");
  if (num_kv_heads < 1) return fail(TACO_ERR_INVALID_ARG, "num_kv_heads must be >= 1");
  if (head_dim != 64 && head_dim != 128) return fail(TACO_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!is_pow2(block_size) || block_size < 8 || block_size > 256)
    return fail(TACO_ERR_UNSUPPORTED, "block_size must be a power of two in [8, 256]");
  if (num_blocks < 1) return fail(TACO_ERR_INVALID_ARG, "num_blocks must be >= 1");
  if (max_blocks < 1) return fail(TACO_ERR_INVALID_ARG, "max_blocks_per_seq must be >= 1");
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size > INT32_MAX)
    return fail(TACO_ERR_UNSUPPORTED, "num_blocks * num_kv_heads * block_size must fit in int32");
  if (static_cast<int64_t>(max_blocks) * block_size > INT32_MAX)
    return fail(TACO_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size must fit in int32");
  return TACO_OK;
}

}  // namespace

namespace taco {
void set_last_error_message(const char* msg) { g_last_error = msg; }
}  // namespace taco

extern "C" {

int32_t taco_attn_version(void) { return kAbiVersion; }

int32_t taco_attn_last_call_launches(void) { return g_last_launches; }

const char* taco_attn_last_error(void) { return g_last_error.c_str(); }

taco_status taco_attn_set_option(int32_t key, int64_t value) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (key == TACO_OPT_GRID_CTAS) {
    if (value < 0 || value > (1 << 20)) return fail(TACO_ERR_INVALID_ARG, "grid size out of range");
    g_opt_grid = value;
    return TACO_OK;
  }
  if (key == TACO_OPT_KERNEL) {
    if (value < 0 || value > 2) return fail(TACO_ERR_INVALID_ARG, "kernel choice must be 0, 1 or 2");
    g_opt_kernel = value;
    return TACO_OK;
  }
  if (key == TACO_OPT_TEST_STALL) {
    if (value < 0 || value > (1 << 30)) return fail(TACO_ERR_INVALID_ARG, "stall tile must be in [0, 2^30]");
    g_opt_stall = value;
    return TACO_OK;
  }
  if (key == TACO_OPT_L2_PREFETCH) {
    if (value < -1 || value > 64) return fail(TACO_ERR_INVALID_ARG, "prefetch distance must be in [-1, 64]");
    g_opt_prefetch = value;
    return TACO_OK;
  }
  if (key == TACO_OPT_COMBINE) {
    if (value < 0 || value > 2) return fail(TACO_ERR_INVALID_ARG, "combine choice must be 0, 1 or 2");
    g_opt_combine = value;
    return TACO_OK;
  }
  if (key == TACO_OPT_SEG_COST) {
    if (value < -1 || value > 64) return fail(TACO_ERR_INVALID_ARG, "segment cost must be in [-1, 64]");
    g_opt_seg_cost = value;
    return TACO_OK;
  }
  return fail(TACO_ERR_INVALID_ARG, "unknown option key %d", key);
}

// Both attention entry points; k_scale / v_scale non-null selects e4m3 caches.
static taco_status attention_impl(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                                  const float* v_scale, const void* k_new, const void* v_new,
                                  const int32_t* block_tables, const int32_t* context_lens,
                                  const int32_t* num_candidates, const uint32_t* tree_mask_bits, float scale,
                                  void* out, int32_t dtype, int32_t batch, int32_t max_candidates,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, int32_t max_blocks_per_seq, void* stream) {
  const bool kv8 = k_scale != nullptr;
  g_last_launches = 0;
  taco_status st = check_common(dtype, batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks_per_seq);
  if (st != TACO_OK) return st;
  if (num_q_heads < 1 || num_q_heads % num_kv_heads != 0)
    return fail(TACO_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !num_candidates || !tree_mask_bits || !out)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (k_new && (!v_new || !aligned16(k_new) || !aligned16(v_new)))
    return fail(TACO_ERR_INVALID_ARG, "k_new and v_new must be non-null and 16-byte aligned");
  if (kv8 && !v_scale) return fail(TACO_ERR_INVALID_ARG, "null pointer argument (v_scale)");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return fail(TACO_ERR_INVALID_ARG, "q, k_cache, v_cache and out must be 16-byte aligned");
  if (!(scale == scale)) return fail(TACO_ERR_INVALID_ARG, "scale is NaN");
  if (batch == 0) return TACO_OK;
  const int G = num_q_heads / num_kv_heads;
  const int packed = G * max_candidates;
  int64_t opt_kernel = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    opt_kernel = g_opt_kernel;
  }
  // kernel choice: the tcgen05 kernel once the packed (GQA group x candidates) tile is wide enough to
  // keep the tensor cores busy, the mma.sync kernel for narrow tiles. e4m3 caches: the mma.sync kernel
  // exists for head_dim 128 and <= 64 packed rows; everything else goes to the tcgen05 kernel, which
  // widens the codes to f16 once per tile
  const bool tc_possible = G <= 128;
  const bool mma_possible = !kv8 || (head_dim == 128 && packed <= 64);
  bool use_tc = tc_possible && (packed >= 48 || !mma_possible);
  if (opt_kernel == 1) {
    if (!mma_possible)
      return fail(TACO_ERR_UNSUPPORTED, "e4m3 caches on the mma.sync path need head_dim 128 and G * C <= 64");
    use_tc = false;
  }
  if (opt_kernel == 2) use_tc = true;
  if (use_tc && !tc_possible)
    return fail(TACO_ERR_UNSUPPORTED, "tensor-core path needs num_q_heads / num_kv_heads <= 128");
  if (!use_tc && !mma_possible)
    return fail(TACO_ERR_UNSUPPORTED, "e4m3 caches: no kernel for num_q_heads / num_kv_heads > 128 with this shape");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);

  std::lock_guard<std::mutex> lk(g_mu);
  int rows, row_groups, cands_per_group = 0;
  if (use_tc) {
    cands_per_group = std::min(max_candidates, 128 / G);
    row_groups = (max_candidates + cands_per_group - 1) / cands_per_group;
    rows = 128;
  } else {
    rows = taco::mma_rows_per_unit(packed);
    row_groups = (packed + rows - 1) / rows;
  }
  const int64_t units = static_cast<int64_t>(batch) * num_kv_heads * row_groups;

  int sms = 0;
  st = sm_count_of(dev, &sms);
  if (st != TACO_OK) return st;
  int grid = static_cast<int>(g_opt_grid);
  if (grid == 0) grid = (use_tc ? 1 : taco::mma_ctas_per_sm(rows)) * sms;
  const size_t slots = 2 * static_cast<size_t>(grid);
  // e4m3 caches with bf16 queries on the tcgen05 path: f16 query rows and their scales in the workspace
  const bool q_convert = use_tc && kv8 && dtype == TACO_DTYPE_BF16;
  const int64_t q_rows = static_cast<int64_t>(batch) * max_candidates * num_q_heads;
  const size_t q16_bytes = q_convert ? round_up(static_cast<size_t>(q_rows) * head_dim * 2, 256) : 0;
  const size_t q_ws = q_convert ? q16_bytes + static_cast<size_t>(q_rows) * 4 : 0;
  Workspace* wp = nullptr;
  st = ensure_workspace(dev, stream, static_cast<size_t>(units), slots * rows, slots * rows * head_dim, &wp, q_ws);
  if (st != TACO_OK) return st;
  Workspace& w = *wp;

  const int tile = use_tc ? taco::tc_tile_keys() : taco::mma_tile_keys(rows, kv8);
  const int rpc = block_size < tile ? block_size : tile;
  const int64_t cache_rows = static_cast<int64_t>(num_blocks) * num_kv_heads * block_size;
  const bool raw_rows = use_tc && kv8;
  CUtensorMap tk, tv, tq;
  st = make_cache_map(&tk, k_cache, dtype, head_dim, cache_rows, rpc, kv8, raw_rows);
  if (st != TACO_OK) return st;
  st = make_cache_map(&tv, v_cache, dtype, head_dim, cache_rows, rpc, kv8, raw_rows);
  if (st != TACO_OK) return st;
  if (use_tc) {
    const void* qsrc = q_convert ? static_cast<const void*>(w.qbuf) : q;
    const int qdtype = kv8 ? TACO_DTYPE_F16 : dtype;
    st = make_query_map(&tq, qsrc, qdtype, head_dim, num_q_heads, static_cast<int64_t>(batch) * max_candidates, G,
                        cands_per_group);
    if (st != TACO_OK) return st;
  }

  taco::VerifyParams p{};
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.num_candidates = num_candidates;
  p.tree_mask_bits = tree_mask_bits;
  p.part_o = w.part_o;
  p.part_lse = w.part_lse;
  p.counters = w.counters;
  p.error_word = w.error_word;
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
  if (g_opt_stall > 0 && !use_tc) {
    p.stall_tile = static_cast<int>(g_opt_stall);
    p.wait_limit_ns = 20000000ull;  // 20 ms
  }
  // Split units with many pieces (few units against many CTAs, such as a handful of long sequences)
  // are merged by a separate combine kernel, one warp per output row, instead of serially by the last
  // CTA to finish each unit at the end of the verify.
  p.defer_merge = (g_opt_combine == 2 || (g_opt_combine == 0 && !use_tc && units * 4 <= grid)) ? 1 : 0;
  p.seg_cost = static_cast<int>(g_opt_seg_cost >= 0 ? g_opt_seg_cost
                                : (use_tc ? taco::tc_seg_cost(cands_per_group * G, kv8) : taco::mma_seg_cost(rows)));
  p.l2_prefetch_tiles = static_cast<int>(
      g_opt_prefetch >= 0 ? g_opt_prefetch : (use_tc ? taco::kTcPrefetchTiles : taco::kMmaPrefetchTiles));
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.q_scale = q_convert ? reinterpret_cast<const float*>(w.qbuf + q16_bytes) : nullptr;
  if (k_new) {
    // fused append where the kernel supports it (mma.sync, <= 16 rows; with e4m3 caches it quantises
    // as the append kernel does); otherwise the append kernel runs first on the same stream
    if (!use_tc && rows <= 16) {
      p.k_new = k_new;
      p.v_new = v_new;
      p.k_cache = const_cast<void*>(k_cache);
      p.v_cache = const_cast<void*>(v_cache);
    } else {
      taco::AppendArgs a{k_new, v_new, block_tables, nullptr, const_cast<void*>(k_cache), const_cast<void*>(v_cache),
                         w.error_word, batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks,
                         max_blocks_per_seq, dtype, context_lens, num_candidates};
      e = kv8 ? taco::launch_append_e4m3(a, k_scale, v_scale, static_cast<cudaStream_t>(stream))
              : taco::launch_append(a, static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
      ++g_last_launches;
      // unless a query conversion runs in between, the verify follows the append directly and may
      // read everything but the appended slots before the append ends
      p.late_wait = q_convert ? 0 : 1;
    }
  }
  // after the append (a plain launch: it starts once the append has finished, and the verify's
  // dependency wait then covers both)
  if (q_convert) {
    e = taco::launch_q_to_f16(q, w.qbuf, reinterpret_cast<float*>(w.qbuf + q16_bytes), q_rows, head_dim,
                              static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "query conversion launch");
    ++g_last_launches;
  }

  if (use_tc)
    e = taco::launch_verify_tc(tk, tv, tq, p, dtype, grid, static_cast<cudaStream_t>(stream));
  else
    e = taco::launch_verify_mma(tk, tv, p, dtype, grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "verify kernel launch");
  ++g_last_launches;
  if (p.defer_merge) {
    e = taco::launch_combine_split(p, dtype, grid, use_tc, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
    ++g_last_launches;
  }
  return TACO_OK;
}

taco_status paged_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 const int32_t* num_candidates, const uint32_t* tree_mask_bits, float scale,
                                 void* out, int32_t dtype, int32_t batch, int32_t max_candidates,
                                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t num_blocks, int32_t max_blocks_per_seq, void* stream) {
  return attention_impl(q, k_cache, v_cache, nullptr, nullptr, nullptr, nullptr, block_tables, context_lens,
                        num_candidates, tree_mask_bits, scale, out, dtype, batch, max_candidates, num_q_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, stream);
}

taco_status paged_tree_attention_append(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                        void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                                        const int32_t* num_candidates, const uint32_t* tree_mask_bits, float scale,
                                        void* out, int32_t dtype, int32_t batch, int32_t max_candidates,
                                        int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                        void* stream) {
  if (!k_new || !v_new) return fail(TACO_ERR_INVALID_ARG, "null pointer argument (k_new / v_new)");
  return attention_impl(q, k_cache, v_cache, nullptr, nullptr, k_new, v_new, block_tables, context_lens,
                        num_candidates, tree_mask_bits, scale, out, dtype, batch, max_candidates, num_q_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, stream);
}

taco_status paged_tree_attention_e4m3(const void* q, const void* k_cache, const void* v_cache,
                                      const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                      const int32_t* context_lens, const int32_t* num_candidates,
                                      const uint32_t* tree_mask_bits, float scale, void* out, int32_t dtype,
                                      int32_t batch, int32_t max_candidates, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                      int32_t num_blocks, int32_t max_blocks_per_seq, void* stream) {
  if (!k_scale || !v_scale) return fail(TACO_ERR_INVALID_ARG, "null pointer argument (k_scale / v_scale)");
  return attention_impl(q, k_cache, v_cache, k_scale, v_scale, nullptr, nullptr, block_tables, context_lens,
                        num_candidates, tree_mask_bits, scale, out, dtype, batch, max_candidates, num_q_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, stream);
}

taco_status paged_tree_attention_append_e4m3(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                             void* v_cache, const float* k_scale, const float* v_scale,
                                             const int32_t* block_tables, const int32_t* context_lens,
                                             const int32_t* num_candidates, const uint32_t* tree_mask_bits,
                                             float scale, void* out, int32_t dtype, int32_t batch,
                                             int32_t max_candidates, int32_t num_q_heads, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                             int32_t max_blocks_per_seq, void* stream) {
  if (!k_new || !v_new) return fail(TACO_ERR_INVALID_ARG, "null pointer argument (k_new / v_new)");
  if (!k_scale || !v_scale) return fail(TACO_ERR_INVALID_ARG, "null pointer argument (k_scale / v_scale)");
  return attention_impl(q, k_cache, v_cache, k_scale, v_scale, k_new, v_new, block_tables, context_lens,
                        num_candidates, tree_mask_bits, scale, out, dtype, batch, max_candidates, num_q_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, stream);
}

taco_status paged_kv_append(const void* k_new, const void* v_new, const int32_t* block_tables,
                            const int32_t* slot_offsets, void* k_cache, void* v_cache, int32_t dtype,
                            int32_t batch, int32_t max_candidates, int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq, void* stream) {
  taco_status st = check_common(dtype, batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks_per_seq);
  if (st != TACO_OK) return st;
  if (!k_new || !v_new || !block_tables || !slot_offsets || !k_cache || !v_cache)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(TACO_ERR_INVALID_ARG, "k_new, v_new, k_cache and v_cache must be 16-byte aligned");
  if (batch == 0) return TACO_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  uint32_t* err = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace* wp = nullptr;
    st = ensure_workspace(dev, stream, 0, 0, 0, &wp);
    if (st != TACO_OK) return st;
    err = wp->error_word;
  }
  taco::AppendArgs a{k_new, v_new, block_tables, slot_offsets, k_cache, v_cache, err,
                     batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq};
  e = taco::launch_append(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  return TACO_OK;
}

taco_status paged_kv_append_e4m3(const void* k_new, const void* v_new, const int32_t* block_tables,
                                 const int32_t* slot_offsets, const float* k_scale, const float* v_scale,
                                 void* k_cache, void* v_cache, int32_t dtype, int32_t batch,
                                 int32_t max_candidates, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
                                 void* stream) {
  taco_status st = check_common(dtype, batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks_per_seq);
  if (st != TACO_OK) return st;
  if (!k_new || !v_new || !block_tables || !slot_offsets || !k_scale || !v_scale || !k_cache || !v_cache)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(TACO_ERR_INVALID_ARG, "k_new, v_new, k_cache and v_cache must be 16-byte aligned");
  if (batch == 0) return TACO_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  uint32_t* err = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace* wp = nullptr;
    st = ensure_workspace(dev, stream, 0, 0, 0, &wp);
    if (st != TACO_OK) return st;
    err = wp->error_word;
  }
  taco::AppendArgs a{k_new, v_new, block_tables, slot_offsets, k_cache, v_cache, err,
                     batch, max_candidates, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                     dtype};
  e = taco::launch_append_e4m3(a, k_scale, v_scale, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  return TACO_OK;
}

// Error word of (the current device, `stream`) (creates the workspace's header on first use).
static taco_status stream_error_word(void* stream, uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace* wp = nullptr;
  taco_status st = ensure_workspace(dev, stream, 0, 0, 0, &wp);
  if (st != TACO_OK) return st;
  *out = wp->error_word;
  return TACO_OK;
}

taco_status tree_mask_from_parents(const int32_t* parents, const int32_t* num_candidates, int32_t batch,
                                   int32_t max_candidates, uint32_t* mask_out, void* stream) {
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (max_candidates < 1 || max_candidates > 32)
    return fail(TACO_ERR_UNSUPPORTED, "max_candidates must be in 1..32 (one mask bit per candidate)");
  if (!parents || !num_candidates || !mask_out) return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (batch == 0) return TACO_OK;
  uint32_t* err = nullptr;
  taco_status st = stream_error_word(stream, &err);
  if (st != TACO_OK) return st;
  taco::MaskArgs a{parents, num_candidates, mask_out, err, batch, max_candidates};
  cudaError_t e = taco::launch_tree_masks(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tree mask kernel launch");
  return TACO_OK;
}

taco_status logits_argmax(const void* logits, int32_t dtype, int64_t rows, int32_t vocab, int32_t* out_index,
                          void* stream) {
  if (dtype != TACO_DTYPE_F16 && dtype != TACO_DTYPE_BF16) return fail(TACO_ERR_INVALID_ARG, "dtype must be f16 or bf16");
  if (rows < 0 || vocab < 1) return fail(TACO_ERR_INVALID_ARG, "need rows >= 0 and vocab >= 1");
  if (rows > 0x7fffffff) return fail(TACO_ERR_UNSUPPORTED, "at most 2^31 - 1 rows per call");
  if (!logits || !out_index) return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (rows == 0) return TACO_OK;
  cudaError_t e = taco::launch_argmax(logits, dtype, rows, vocab, out_index, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "argmax kernel launch");
  return TACO_OK;
}

taco_status tree_greedy_accept(const int32_t* target_argmax, const int32_t* candidate_tokens,
                               const int32_t* parents, const int32_t* num_candidates, const int32_t* context_lens,
                               int32_t batch, int32_t max_candidates, int32_t* accept_len, int32_t* accepted_path,
                               int32_t* bonus_token, int32_t* slot_offsets_out, void* stream) {
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (max_candidates < 1 || max_candidates > 32)
    return fail(TACO_ERR_UNSUPPORTED, "max_candidates must be in 1..32 (one lane per candidate)");
  if (!target_argmax || !candidate_tokens || !parents || !num_candidates || !context_lens || !accept_len ||
      !accepted_path || !bonus_token || !slot_offsets_out)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (batch == 0) return TACO_OK;
  uint32_t* err = nullptr;
  taco_status st = stream_error_word(stream, &err);
  if (st != TACO_OK) return st;
  taco::AcceptArgs a{target_argmax, candidate_tokens, parents, num_candidates, context_lens, accept_len,
                     accepted_path, bonus_token, slot_offsets_out, err, batch, max_candidates};
  cudaError_t e = taco::launch_accept(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "accept kernel launch");
  return TACO_OK;
}

static taco_status prefix_common(const int32_t* tokens, const int32_t* seq_starts, const void* slot_keys,
                                 const void* slot_nodes, int64_t capacity, const void* node_parent,
                                 const void* node_depth, const void* node_tokens, const void* out_blocks,
                                 int32_t batch, int32_t block_size, int32_t num_blocks, int32_t max_blocks,
                                 void* stream, uint32_t** err) {
  if (!tokens || !seq_starts || !slot_keys || !slot_nodes || !node_parent || !node_depth || !node_tokens ||
      !out_blocks)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if ((reinterpret_cast<uintptr_t>(slot_keys) & 7u) != 0) return fail(TACO_ERR_INVALID_ARG, "slot_keys must be 8-byte aligned");
  if (capacity < 2 || (capacity & (capacity - 1)) != 0) return fail(TACO_ERR_INVALID_ARG, "capacity must be a power of two >= 2");
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (block_size < 1 || block_size > 1024) return fail(TACO_ERR_UNSUPPORTED, "block_size must be in [1, 1024]");
  if (num_blocks < 1) return fail(TACO_ERR_INVALID_ARG, "num_blocks must be >= 1");
  if (max_blocks < 1) return fail(TACO_ERR_INVALID_ARG, "max_blocks_per_seq must be >= 1");
  if (batch == 0) return TACO_OK;
  return stream_error_word(stream, err);
}

taco_status prefix_cache_lookup(const int32_t* tokens, const int32_t* seq_starts, const uint64_t* slot_keys,
                                const int32_t* slot_nodes, int64_t capacity, const int32_t* node_parent,
                                const int32_t* node_depth, const int32_t* node_tokens, int32_t* out_blocks,
                                int32_t* out_matched, int32_t batch, int32_t block_size, int32_t num_blocks,
                                int32_t max_blocks_per_seq, void* stream) {
  if (!out_matched) return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  uint32_t* err = nullptr;
  taco_status st = prefix_common(tokens, seq_starts, slot_keys, slot_nodes, capacity, node_parent, node_depth,
                                 node_tokens, out_blocks, batch, block_size, num_blocks, max_blocks_per_seq, stream,
                                 &err);
  if (st != TACO_OK || batch == 0) return st;
  cudaError_t e = taco::launch_prefix_cache(false, tokens, seq_starts, nullptr, const_cast<uint64_t*>(slot_keys),
                                            const_cast<int32_t*>(slot_nodes), capacity, const_cast<int32_t*>(node_parent),
                                            const_cast<int32_t*>(node_depth), const_cast<int32_t*>(node_tokens),
                                            out_blocks, out_matched, err, batch, block_size, num_blocks,
                                            max_blocks_per_seq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefix lookup launch");
  return TACO_OK;
}

taco_status prefix_cache_insert(const int32_t* tokens, const int32_t* seq_starts, const int32_t* block_tables,
                                uint64_t* slot_keys, int32_t* slot_nodes, int64_t capacity, int32_t* node_parent,
                                int32_t* node_depth, int32_t* node_tokens, int32_t* out_blocks,
                                int32_t* out_inserted, int32_t batch, int32_t block_size, int32_t num_blocks,
                                int32_t max_blocks_per_seq, void* stream) {
  if (!block_tables) return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  uint32_t* err = nullptr;
  taco_status st = prefix_common(tokens, seq_starts, slot_keys, slot_nodes, capacity, node_parent, node_depth,
                                 node_tokens, out_blocks, batch, block_size, num_blocks, max_blocks_per_seq, stream,
                                 &err);
  if (st != TACO_OK || batch == 0) return st;
  cudaError_t e = taco::launch_prefix_cache(true, tokens, seq_starts, block_tables, slot_keys, slot_nodes, capacity,
                                            node_parent, node_depth, node_tokens, out_blocks, out_inserted, err, batch,
                                            block_size, num_blocks, max_blocks_per_seq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefix insert launch");
  return TACO_OK;
}

taco_status lookahead_propose(const int32_t* history, const int32_t* hist_starts, const int32_t* global_tokens,
                              int64_t global_len, const int32_t* copy_len, int32_t max_match, int32_t batch,
                              int32_t max_candidates, int32_t* tokens_out, int32_t* parents_out,
                              int32_t* num_candidates_out, void* stream) {
  if (!history || !hist_starts || !copy_len || !tokens_out || !parents_out || !num_candidates_out)
    return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (global_len < 0 || global_len > INT32_MAX) return fail(TACO_ERR_INVALID_ARG, "global_len must be in [0, 2^31)");
  if (global_len > 0 && !global_tokens) return fail(TACO_ERR_INVALID_ARG, "null global_tokens with global_len > 0");
  if (max_match < 1 || max_match > 16) return fail(TACO_ERR_UNSUPPORTED, "max_match must be in [1, 16]");
  if (max_candidates < 1 || max_candidates > 32) return fail(TACO_ERR_UNSUPPORTED, "max_candidates must be in [1, 32]");
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (batch == 0) return TACO_OK;
  uint32_t* err = nullptr;
  taco_status st = stream_error_word(stream, &err);
  if (st != TACO_OK) return st;
  cudaError_t e = taco::launch_lookahead_propose(history, hist_starts, global_len > 0 ? global_tokens : nullptr,
                                                 global_len, copy_len, max_match, batch, max_candidates, tokens_out,
                                                 parents_out, num_candidates_out, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lookahead kernel launch");
  return TACO_OK;
}

taco_status lookahead_update_copy_len(const int32_t* accept_len, const int32_t* num_proposed, float* hit,
                                      int32_t* copy_len, int32_t batch, int32_t copy_max, float alpha,
                                      int32_t batch_ref, void* stream) {
  if (!accept_len || !num_proposed || !hit || !copy_len) return fail(TACO_ERR_INVALID_ARG, "null pointer argument");
  if (batch < 0) return fail(TACO_ERR_INVALID_ARG, "batch must be >= 0");
  if (copy_max < 1) return fail(TACO_ERR_INVALID_ARG, "copy_max must be >= 1");
  if (!(alpha >= 0.f && alpha <= 1.f)) return fail(TACO_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (batch_ref < 1) return fail(TACO_ERR_INVALID_ARG, "batch_ref must be >= 1");
  if (batch == 0) return TACO_OK;
  cudaError_t e = taco::launch_copy_len_update(accept_len, num_proposed, hit, copy_len, batch, copy_max, alpha,
                                               batch_ref, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "copy_len kernel launch");
  return TACO_OK;
}

taco_status taco_attn_check_device(void* stream, uint32_t* bits_out) {
  if (bits_out) *bits_out = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TACO_ERR_UNSUPPORTED, "device index %d too large", dev);
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_ws.find(std::make_pair(dev, reinterpret_cast<uintptr_t>(stream)));
  if (it == g_ws.end() || !it->second.base) return TACO_OK;
  Workspace& w = it->second;
  uint32_t bits = 0;
  e = cudaMemcpy(&bits, w.error_word, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (error word)");
  if (bits_out) *bits_out = bits;
  if (bits == 0) return TACO_OK;
  cudaMemset(w.error_word, 0, 4);
  if (bits & TACO_DEVERR_WAIT_TIMEOUT) cudaMemset(w.counters, 0, w.counters_cap * 4);
  return fail(TACO_ERR_DEVICE_CHECK, "device range check failed: bits 0x%x%s%s%s%s%s%s%s", bits,
              (bits & TACO_DEVERR_BLOCK_ID) ? " [block id out of range]" : "",
              (bits & TACO_DEVERR_CONTEXT_LEN) ? " [context length out of range]" : "",
              (bits & TACO_DEVERR_NUM_CAND) ? " [candidate count out of range]" : "",
              (bits & TACO_DEVERR_SLOT) ? " [slot out of range]" : "",
              (bits & TACO_DEVERR_WAIT_TIMEOUT) ? " [pipeline wait timed out]" : "",
              (bits & TACO_DEVERR_PARENT) ? " [parent index out of range]" : "",
              (bits & TACO_DEVERR_TABLE_FULL) ? " [prefix table full]" : "");
}

void taco_attn_release_workspace(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ws) {
    if (!kv.second.base) continue;
    cudaSetDevice(kv.first.first);
    cudaFree(kv.second.base);
  }
  g_ws.clear();
  cudaSetDevice(cur);
}

}  // extern "C"
