// C ABI of libmla_decode.so: argument validation, TMA tensor-map encoding and
// kernel launches. See include/mla_decode.h for the contract of each call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/mla_decode.h"
#include "mla_common.cuh"
#include "mla_launch.h"

namespace {

thread_local std::string g_last_error;
thread_local unsigned long long g_timeout_ns = 1000ull * 1000 * 1000;
long long* g_trace = nullptr;   // instrumented builds: device buffer for phase stamps

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MLA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
  int device = -1;
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
  int max_clusters[2][2] = {{0, 0}, {0, 0}};   // 2-CTA clusters that fit: [fp8][128-row tiles]
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

int device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MLA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.device != dev) {
    DeviceInfo n;
    n.device = dev;
    if ((e = cudaDeviceGetAttribute(&n.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    if ((e = cudaDeviceGetAttribute(&n.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(cc major)");
    if ((e = cudaDeviceGetAttribute(&n.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(cc minor)");
    if (n.cc_major != 10 || n.cc_minor != 0)
      return fail(MLA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev,
                  n.cc_major, n.cc_minor);
    for (int f = 0; f < 2; ++f) {
      for (int v = 0; v < 2; ++v) {
        if ((e = mla::decode_max_active_clusters(v == 0 ? 64 : 128, f == 1, &n.max_clusters[f][v])) != cudaSuccess)
          return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
        if (n.max_clusters[f][v] < 1)
          return fail(MLA_ERR_UNSUPPORTED, "no 2-CTA cluster of the decode kernel fits");
      }
    }
    d = n;
  }
  *out = d;
  return MLA_OK;
}

// Query rows per tile: a step with at most 64 rows (q_len * heads) uses the
// 64-row kernel variant, whose smaller Q tile leaves room for a deeper KV ring.
int tile_rows_of(int q_len, int heads) { return q_len * heads <= 64 ? 64 : 128; }

int row_tiles_of(int q_len, int heads) {
  const int tr = tile_rows_of(q_len, heads);
  return (q_len * heads + tr - 1) / tr;
}

// Clusters per row tile the grid is sized for (the planner may use fewer).
int clusters_per_tile(const DeviceInfo& d, int q_len, int heads, int kv_dtype) {
  const int c = d.max_clusters[kv_dtype == MLA_KV_FP8_E4M3 ? 1 : 0][tile_rows_of(q_len, heads) == 64 ? 0 : 1] /
                row_tiles_of(q_len, heads);
  return c < 1 ? 1 : c;
}

// Query rows of the one-sequence prefix pass of a cascade step (the union of
// the batch's rows): at most 64 row tiles, so that every row tile still gets
// a cluster.
constexpr int kWideRows = 8192;

int check_shape(int batch, int max_pages, int q_len, int heads, int kv_dtype, bool wide = false) {
  if (batch < 0) return fail(MLA_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", batch);
  if (max_pages < 1) return fail(MLA_ERR_INVALID_ARG, "max_pages_per_seq must be >= 1 (got %d)", max_pages);
  if (max_pages > (1 << 24)) return fail(MLA_ERR_UNSUPPORTED, "max_pages_per_seq %d too large", max_pages);
  if (q_len < 1 || q_len > 4) return fail(MLA_ERR_UNSUPPORTED, "q_len must be in [1, 4] (got %d)", q_len);
  if (wide) {   // internal: the prefix pass of a cascade step, every row a single query token
    if (q_len != 1 || heads < 1 || heads > kWideRows)
      return fail(MLA_ERR_UNSUPPORTED, "cascade: batch * q_len * heads must be in [1, %d] (got %d)", kWideRows, heads);
  } else {
    if (heads < 1 || heads > 128) return fail(MLA_ERR_UNSUPPORTED, "heads must be in [1, 128] (got %d)", heads);
    if (q_len * heads > 512) return fail(MLA_ERR_UNSUPPORTED, "q_len * heads must be <= 512");
  }
  if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_FP8_E4M3)
    return fail(MLA_ERR_INVALID_ARG, "kv_dtype %d is not an mla_kv_dtype", kv_dtype);
  if (static_cast<long long>(batch) * q_len * heads > (1ll << 30))
    return fail(MLA_ERR_UNSUPPORTED, "batch * q_len * heads too large");
  // The planner's cost line (n_b + 2 units per sequence) and every position on
  // it, plus one payload past its end, must fit in int32.
  if (static_cast<long long>(batch) * (max_pages + mla::kSeqOverhead) > (1ll << 30))
    return fail(MLA_ERR_UNSUPPORTED, "batch * (max_pages_per_seq + %d) exceeds 2^30", mla::kSeqOverhead);
  return MLA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Pointers already found to be device or managed memory, per device (a small
// ring: a decode loop passes the same few buffers every step, and each
// cudaPointerGetAttributes call costs host time on the launch path).
struct PtrCache {
  static constexpr int kSize = 32;
  const void* ptr[kSize] = {};
  int next = 0;
};
std::mutex g_ptr_mu;
PtrCache g_ptr_cache[64];

int check_device_ptr(const void* p, const char* name) {
  int dev = 0;
  const bool have_dev = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64;
  if (have_dev) {
    std::lock_guard<std::mutex> lk(g_ptr_mu);
    const PtrCache& c = g_ptr_cache[dev];
    for (int i = 0; i < PtrCache::kSize; ++i)
      if (c.ptr[i] == p) return MLA_OK;
  }
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MLA_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorName(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(MLA_ERR_INVALID_ARG, "%s must be device or managed memory", name);
  if (have_dev) {
    std::lock_guard<std::mutex> lk(g_ptr_mu);
    PtrCache& c = g_ptr_cache[dev];
    c.ptr[c.next] = p;
    c.next = (c.next + 1) % PtrCache::kSize;
  }
  return MLA_OK;
}

// Encoded TMA descriptors, keyed by everything that goes into them, per
// device: a decode loop re-encodes the same few maps every step otherwise.
struct MapKey {
  int device, kind;          // kind: which map of the run (query rope, cache, cache rope; x dtype)
  const void* base;
  unsigned long long dim1, dim2;
  bool operator==(const MapKey& o) const {
    return device == o.device && kind == o.kind && base == o.base && dim1 == o.dim1 && dim2 == o.dim2;
  }
};
struct MapCache {
  static constexpr int kSize = 16;
  MapKey key[kSize];
  CUtensorMap map[kSize];
  bool used[kSize] = {};
  int next = 0;
};
std::mutex g_map_mu;
MapCache g_map_cache;

bool map_lookup(const MapKey& k, CUtensorMap* out) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  for (int i = 0; i < MapCache::kSize; ++i) {
    if (g_map_cache.used[i] && g_map_cache.key[i] == k) {
      *out = g_map_cache.map[i];
      return true;
    }
  }
  return false;
}

void map_store(const MapKey& k, const CUtensorMap& m) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  const int i = g_map_cache.next;
  g_map_cache.key[i] = k;
  g_map_cache.map[i] = m;
  g_map_cache.used[i] = true;
  g_map_cache.next = (i + 1) % MapCache::kSize;
}

// The cluster budget of the last plan enqueued on each workspace, with the
// shape it was planned for. A run on a workspace found here with the same shape
// lets the decode kernel derive that plan itself (small batches), instead of
// waiting for the planner kernel; a run on any other workspace reads the
// planner's output as usual.
struct PlanRecord {
  const void* ws = nullptr;
  int c_use = 0, batch = 0, max_pages = 0, q_len = 0, heads = 0, kv_dtype = 0;
  bool wide = false;
  bool same_shape(int b, int mp, int ql, int h, int kd, bool wd) const {
    return batch == b && max_pages == mp && q_len == ql && heads == h && kv_dtype == kd && wide == wd;
  }
};
constexpr int kPlanRecords = 64;
std::mutex g_plan_mu;
PlanRecord g_plan_rec[kPlanRecords];
int g_plan_next = 0;

void plan_record(const PlanRecord& r) {
  std::lock_guard<std::mutex> lk(g_plan_mu);
  for (auto& e : g_plan_rec) {
    if (e.ws == r.ws) {
      e = r;
      return;
    }
  }
  g_plan_rec[g_plan_next] = r;
  g_plan_next = (g_plan_next + 1) % kPlanRecords;
}

// The recorded cluster budget for (ws, shape), or 0 when there is none.
int plan_c_use(const void* ws, int batch, int max_pages, int q_len, int heads, int kv_dtype, bool wide) {
  std::lock_guard<std::mutex> lk(g_plan_mu);
  for (const auto& e : g_plan_rec)
    if (e.ws == ws) return e.same_shape(batch, max_pages, q_len, heads, kv_dtype, wide) ? e.c_use : 0;
  return 0;
}

}  // namespace

namespace mla {
int set_last_error(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}
}  // namespace mla

extern "C" {

const char* mla_get_last_error(void) { return g_last_error.c_str(); }

const char* mla_version(void) { return "mla_decode 0.1 (sm_100a)"; }

#ifdef MLA_TRACE
// Instrumented builds only: device buffer of 6144 int64 for phase stamps.
MLA_API void mla_debug_set_trace(long long* device_buffer) { g_trace = device_buffer; }
#endif

int mla_set_wait_timeout_ns(uint64_t timeout_ns) {
  g_timeout_ns = static_cast<unsigned long long>(timeout_ns);
  return MLA_OK;
}

}  // extern "C"

namespace {

int plan_impl(const int32_t* seqlens, const int32_t* block_table, int64_t num_pages, int batch,
              int max_pages_per_seq, int q_len, int heads, int kv_dtype, int sm_budget, void* workspace,
              size_t* workspace_bytes, int* num_splits, void* stream, bool wide) {
  g_last_error.clear();
  if (!workspace_bytes) return fail(MLA_ERR_INVALID_ARG, "workspace_bytes is NULL");
  int st = check_shape(batch, max_pages_per_seq, q_len, heads, kv_dtype, wide);
  if (st != MLA_OK) return st;
  if (sm_budget < 0) return fail(MLA_ERR_INVALID_ARG, "sm_budget must be >= 0 (got %d)", sm_budget);
  if (block_table) {
    if (!aligned(block_table, 4)) return fail(MLA_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
    if (num_pages < 1 || num_pages > 0x7FFFFFFFll)
      return fail(MLA_ERR_INVALID_ARG, "num_pages must be in [1, 2^31-1] when block_table is given (got %lld)",
                  (long long)num_pages);
  }
  DeviceInfo d;
  if ((st = device_info(&d)) != MLA_OK) return st;
  const int rt = row_tiles_of(q_len, heads);
  const int c_max = clusters_per_tile(d, q_len, heads, kv_dtype);
  const mla::WsLayout w = mla::ws_layout(batch, rt, c_max);
  const size_t capacity = *workspace_bytes;
  *workspace_bytes = w.total;
  if (num_splits) *num_splits = w.max_slots;
  if (!workspace) return MLA_OK;
  if (!aligned(workspace, 256)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (capacity < w.total)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", capacity, w.total);
  if (batch > 0) {
    if (!seqlens) return fail(MLA_ERR_INVALID_ARG, "seqlens is NULL");
    if (!aligned(seqlens, 4)) return fail(MLA_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
    if ((st = check_device_ptr(seqlens, "seqlens")) != MLA_OK) return st;
    if (block_table && (st = check_device_ptr(block_table, "block_table")) != MLA_OK) return st;
  }
  if ((st = check_device_ptr(workspace, "workspace")) != MLA_OK) return st;
  int c_use = c_max;
  if (sm_budget > 0) {
    c_use = (sm_budget / 2) / rt;
    if (c_use < 1) c_use = 1;
    if (c_use > c_max) c_use = c_max;
  }
  mla::PlanParams pp;
  pp.seqlens = seqlens;
  pp.block_table = batch > 0 ? block_table : nullptr;
  pp.num_pages = num_pages;
  // A batch the decode kernel plans itself, at 64 rows per tile, gets the
  // one-warp planner: it and its checking warps fit on SMs beside the decode
  // CTAs, which start without waiting for them. (A 128-row decode CTA holds all
  // of an SM's registers, so there the wider planner, done sooner, is better.)
  pp.warp_plan = (batch >= 1 && batch <= mla::kSelfPlanMaxBatch && tile_rows_of(q_len, heads) == 64) ? 1 : 0;
  pp.check_ctas = 0;
  if (pp.block_table) {   // one checking CTA per kCheckEntriesPerCta (warp: kCheckEntriesPerWarp) entries
    const long long per = pp.warp_plan ? mla::kCheckEntriesPerWarp : mla::kCheckEntriesPerCta;
    const long long entries = static_cast<long long>(batch) * max_pages_per_seq;
    const long long g = (entries + per - 1) / per;
    pp.check_ctas = static_cast<int>(g < 1 ? 1 : (g > mla::kMaxCheckCtas ? mla::kMaxCheckCtas : g));
  }
  pp.ws = static_cast<int32_t*>(workspace);
  pp.batch = batch;
  pp.max_pages = max_pages_per_seq;
  pp.q_len = q_len;
  pp.row_tiles = rt;
  pp.rows = q_len * heads;
  pp.c_max = c_max;
  pp.c_use = c_use;
  pp.trace = g_trace;
  cudaError_t e = mla::launch_plan(pp, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "planner launch");
  PlanRecord rec;
  rec.ws = workspace;
  rec.c_use = c_use;
  rec.batch = batch;
  rec.max_pages = max_pages_per_seq;
  rec.q_len = q_len;
  rec.heads = heads;
  rec.kv_dtype = kv_dtype;
  rec.wide = wide;
  plan_record(rec);
  return MLA_OK;
}

int run_impl(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype, const int32_t* block_table,
             const int32_t* seqlens, void* out, float* lse, int batch, int max_pages_per_seq, int q_len, int heads,
             float scale, void* workspace, size_t workspace_bytes, int phases, void* stream, bool wide) {
  g_last_error.clear();
  if (phases <= 0 || (phases & ~(MLA_PHASE_ATTEND | MLA_PHASE_COMBINE)) != 0)
    return fail(MLA_ERR_INVALID_ARG, "phases must be a non-empty OR of MLA_PHASE_ATTEND/MLA_PHASE_COMBINE");
  int st = check_shape(batch, max_pages_per_seq, q_len, heads, kv_dtype, wide);
  if (st != MLA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MLA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (num_pages < 1 || num_pages > 0x7FFFFFFFll)
    return fail(MLA_ERR_INVALID_ARG, "num_pages must be in [1, 2^31-1] (got %lld)", (long long)num_pages);
  DeviceInfo d;
  if ((st = device_info(&d)) != MLA_OK) return st;
  const int rt = row_tiles_of(q_len, heads);
  const int c_max = clusters_per_tile(d, q_len, heads, kv_dtype);
  const mla::WsLayout w = mla::ws_layout(batch, rt, c_max);
  if (!workspace) return fail(MLA_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", workspace_bytes, w.total);
  // A split sequence has at most one piece per cluster; the combine kernel
  // handles kCombineMaxSplits pieces. Checked before anything is enqueued.
  if (c_max > mla::kCombineMaxSplits)
    return fail(MLA_ERR_UNSUPPORTED, "%d clusters per row tile exceed the combine limit of %d pieces", c_max,
                mla::kCombineMaxSplits);
  if (batch == 0) return MLA_OK;
  const struct {
    const void* p;
    const char* name;
    size_t align;
  } ptrs[] = {{q, "q", 16},           {kv_cache, "kv_cache", 16}, {block_table, "block_table", 4},
              {seqlens, "seqlens", 4}, {out, "out", 16},           {lse, "lse", 4}};
  for (const auto& x : ptrs) {
    if (!x.p) return fail(MLA_ERR_INVALID_ARG, "%s is NULL", x.name);
    if (!aligned(x.p, x.align)) return fail(MLA_ERR_INVALID_ARG, "%s must be %zu-byte aligned", x.name, x.align);
    if ((st = check_device_ptr(x.p, x.name)) != MLA_OK) return st;
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");

  const int rows = q_len * heads;
  const int tile_rows = tile_rows_of(q_len, heads);
  const bool fp8 = kv_dtype == MLA_KV_FP8_E4M3;
  CUtensorMap tm_q, tm_kv, tm_kv2;
  memset(&tm_kv2, 0, sizeof(tm_kv2));
  int dev = 0;
  cudaGetDevice(&dev);
  // a bf16 cache: each CTA loads only its 32 rope columns (64-byte swizzle)
  const bool narrow_rope = !fp8;
  // Cache keys: map kinds 0-3 query (narrow x tile height), 4/5 bf16 cache
  // latent/rope boxes, 6/7 fp8 cache latent/rope boxes.
  const MapKey kq{dev, (narrow_rope ? 1 : 0) + (tile_rows == 128 ? 2 : 0), q,
                  static_cast<unsigned long long>(batch) * rows, 0};
  if (!map_lookup(kq, &tm_q)) {
    // query rope boxes: [tile_rows x 64 (narrow: 32)] bf16 from column 512 (the
    // latent slice is read directly by the kernel into tensor memory)
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(batch) * rows};
    const cuuint64_t strides[1] = {mla::kDqk * 2};
    const cuuint32_t box[2] = {narrow_rope ? 32u : 64u, static_cast<cuuint32_t>(tile_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, narrow_rope ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(q) failed (%d)", static_cast<int>(r));
    map_store(kq, tm_q);
  }
  const MapKey kkv{dev, fp8 ? 6 : 4, kv_cache, static_cast<unsigned long long>(num_pages), 0};
  const MapKey kkv2{dev, fp8 ? 7 : 5, kv_cache, static_cast<unsigned long long>(num_pages), 0};
  const bool have_kv = map_lookup(kkv, &tm_kv) && map_lookup(kkv2, &tm_kv2);
  if (!have_kv && !fp8) {
    // pages [num_pages][64][576] bf16; boxes of 64 tokens x 64 columns
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(mla::kPage),
                                static_cast<cuuint64_t>(num_pages)};
    const cuuint64_t strides[2] = {mla::kDqk * 2, static_cast<cuuint64_t>(mla::kDqk) * 2 * mla::kPage};
    const cuuint32_t box[3] = {64, mla::kPage, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv_cache), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(kv_cache) failed (%d)", static_cast<int>(r));
    if (narrow_rope) {   // rope boxes of 64 tokens x 32 columns
      const cuuint32_t box_rope[3] = {32, mla::kPage, 1};
      r = enc(&tm_kv2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv_cache), dims, strides, box_rope,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS)
        return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(kv rope) failed (%d)", static_cast<int>(r));
    }
    map_store(kkv, tm_kv);
    map_store(kkv2, tm_kv2);
  } else if (!have_kv) {
    // fp8 pages: 64 x 576 e4m3 codes (row stride 576 B) then 64 fp32 scales;
    // page stride 37,120 B. Latent boxes 64 tokens x 128 codes (128B swizzle),
    // rope boxes 64 tokens x 64 codes (unswizzled 64-byte rows).
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(mla::kPage),
                                static_cast<cuuint64_t>(num_pages)};
    const cuuint64_t strides[2] = {mla::kDqk, static_cast<cuuint64_t>(mla::kFp8PageBytes)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint32_t box_lat[3] = {128, mla::kPage, 1};
    CUresult r = enc(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(kv_cache), dims, strides,
                     box_lat, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(fp8 kv_cache) failed (%d)", static_cast<int>(r));
    const cuuint32_t box_rope[3] = {64, mla::kPage, 1};
    r = enc(&tm_kv2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(kv_cache), dims, strides, box_rope, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(fp8 rope) failed (%d)", static_cast<int>(r));
    map_store(kkv, tm_kv);
    map_store(kkv2, tm_kv2);
  }
  mla::DecodeParams p;
  p.q = q;
  p.kv_cache = kv_cache;
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.ws = static_cast<int32_t*>(workspace);
  p.batch = batch;
  p.max_pages = max_pages_per_seq;
  p.q_len = q_len;
  p.heads = heads;
  p.rows = rows;
  p.row_tiles = rt;
  p.c_max = c_max;
  p.tile_rows = tile_rows;
  p.fp8 = fp8 ? 1 : 0;
  p.num_pages = num_pages;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.c_use = batch >= 1 && batch <= mla::kSelfPlanMaxBatch
                ? plan_c_use(workspace, batch, max_pages_per_seq, q_len, heads, kv_dtype, wide)
                : 0;
  p.self_plan = p.c_use > 0 ? 1 : 0;
  p.timeout_ns = g_timeout_ns;
  p.trace = g_trace;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (phases & MLA_PHASE_ATTEND) {
    e = mla::launch_decode(tm_q, tm_kv, tm_kv2, p, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  }
  if (!(phases & MLA_PHASE_COMBINE)) return MLA_OK;
  mla::CombineParams cp;
  cp.ws = p.ws;
  cp.out = p.out;
  cp.lse = lse;
  cp.batch = batch;
  cp.rows = rows;
  cp.row_tiles = rt;
  cp.c_max = c_max;
  cp.tile_rows = p.tile_rows;
  // A step with no more combine work items than two per SM (its bound: one
  // sequence with at most 74 query rows gives at most rows * 4) gets one CTA per
  // item, which launch_combine spreads over the SMs; larger steps get a
  // persistent grid of four CTAs per SM.
  const long long items_max = static_cast<long long>(batch) * rows * 4;
  cp.grid = items_max <= 2ll * d.sms ? static_cast<int>(items_max) : 4 * d.sms;
  cp.trace = g_trace;
  e = mla::launch_combine(cp, s);
  if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_decode_plan(const int32_t* seqlens, const int32_t* block_table, int64_t num_pages, int batch,
                    int max_pages_per_seq, int q_len, int heads, int kv_dtype, int sm_budget, void* workspace,
                    size_t* workspace_bytes, int* num_splits, void* stream) {
  return plan_impl(seqlens, block_table, num_pages, batch, max_pages_per_seq, q_len, heads, kv_dtype, sm_budget,
                   workspace, workspace_bytes, num_splits, stream, false);
}

int mla_decode_run(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                   const int32_t* block_table, const int32_t* seqlens, void* out, float* lse, int batch,
                   int max_pages_per_seq, int q_len, int heads, float scale, void* workspace,
                   size_t workspace_bytes, void* stream) {
  return run_impl(q, kv_cache, num_pages, kv_dtype, block_table, seqlens, out, lse, batch, max_pages_per_seq, q_len,
                  heads, scale, workspace, workspace_bytes, MLA_PHASE_ATTEND | MLA_PHASE_COMBINE, stream, false);
}

int mla_decode_run_phases(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                          const int32_t* block_table, const int32_t* seqlens, void* out, float* lse, int batch,
                          int max_pages_per_seq, int q_len, int heads, float scale, void* workspace,
                          size_t workspace_bytes, int phases, void* stream) {
  return run_impl(q, kv_cache, num_pages, kv_dtype, block_table, seqlens, out, lse, batch, max_pages_per_seq, q_len,
                  heads, scale, workspace, workspace_bytes, phases, stream, false);
}

int mla_decode_cascade(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                       const int32_t* block_table, const int32_t* seqlens, int prefix_len, void* out, float* lse,
                       int batch, int max_pages_per_seq, int q_len, int heads, float scale, void* workspace,
                       size_t* workspace_bytes, void* stream) {
  g_last_error.clear();
  if (!workspace_bytes) return fail(MLA_ERR_INVALID_ARG, "workspace_bytes is NULL");
  int st = check_shape(batch, max_pages_per_seq, q_len, heads, kv_dtype);
  if (st != MLA_OK) return st;
  if (prefix_len < 0 || prefix_len % mla::kPage != 0 || prefix_len > max_pages_per_seq * mla::kPage)
    return fail(MLA_ERR_INVALID_ARG, "prefix_len must be a multiple of 64 in [0, 64 * max_pages_per_seq] (got %d)",
                prefix_len);
  const long long rows_total = static_cast<long long>(batch) * q_len * heads;
  if (rows_total > kWideRows)
    return fail(MLA_ERR_UNSUPPORTED, "cascade: batch * q_len * heads must be <= %d (got %lld)", kWideRows, rows_total);
  // Workspace: [prefix-pass workspace | suffix-pass workspace | prefix out, lse | suffix out, lse |
  //             cascade words (flag) | prefix length | suffix lengths]
  const int rows = static_cast<int>(rows_total);
  size_t ws_pre = 0, ws_suf = 0;
  if (batch > 0 && (st = plan_impl(nullptr, nullptr, 0, 1, max_pages_per_seq, 1, rows, kv_dtype, 0, nullptr, &ws_pre,
                                   nullptr, stream, true)) != MLA_OK)
    return st;
  if ((st = plan_impl(nullptr, nullptr, 0, batch, max_pages_per_seq, q_len, heads, kv_dtype, 0, nullptr, &ws_suf,
                      nullptr, stream, false)) != MLA_OK)
    return st;
  const size_t o_pre = 0;
  const size_t o_suf = mla::align_up(o_pre + ws_pre, 256);
  const size_t o_out1 = mla::align_up(o_suf + ws_suf, 256);
  const size_t o_lse1 = mla::align_up(o_out1 + static_cast<size_t>(rows) * mla::kDv * 2, 256);
  const size_t o_out2 = mla::align_up(o_lse1 + static_cast<size_t>(rows) * 4, 256);
  const size_t o_lse2 = mla::align_up(o_out2 + static_cast<size_t>(rows) * mla::kDv * 2, 256);
  const size_t o_words = mla::align_up(o_lse2 + static_cast<size_t>(rows) * 4, 256);
  const size_t o_slp = o_words + 256;
  const size_t o_sls = mla::align_up(o_slp + 4, 16);
  const size_t total = mla::align_up(o_sls + 4 * static_cast<size_t>(batch), 256);
  const size_t capacity = *workspace_bytes;
  *workspace_bytes = total;
  if (!workspace) return MLA_OK;
  if (!aligned(workspace, 256)) return fail(MLA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (capacity < total) return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", capacity, total);
  if (batch == 0) return MLA_OK;
  for (const void* x : {static_cast<const void*>(seqlens), static_cast<const void*>(block_table)})
    if (!x || !aligned(x, 4)) return fail(MLA_ERR_INVALID_ARG, "seqlens and block_table must be non-NULL, 4-byte aligned");
  if ((st = check_device_ptr(seqlens, "seqlens")) != MLA_OK) return st;
  if ((st = check_device_ptr(block_table, "block_table")) != MLA_OK) return st;
  char* ws = static_cast<char*>(workspace);
  int32_t* sl_pre = reinterpret_cast<int32_t*>(ws + o_slp);
  int32_t* sl_suf = reinterpret_cast<int32_t*>(ws + o_sls);
  int32_t* cflag = reinterpret_cast<int32_t*>(ws + o_words);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (prefix_len == 0) {   // no shared prefix: an ordinary step into out / lse
    size_t cap = ws_suf;
    if ((st = plan_impl(seqlens, block_table, num_pages, batch, max_pages_per_seq, q_len, heads, kv_dtype, 0, ws,
                        &cap, nullptr, stream, false)) != MLA_OK)
      return st;
    return run_impl(q, kv_cache, num_pages, kv_dtype, block_table, seqlens, out, lse, batch, max_pages_per_seq, q_len,
                    heads, scale, ws, ws_suf, MLA_PHASE_ATTEND | MLA_PHASE_COMBINE, stream, false);
  }
  mla::CascadeParams cp;
  cp.seqlens = seqlens;
  cp.block_table = block_table;
  cp.seqlens_suffix = sl_suf;
  cp.seqlen_prefix = sl_pre;
  cp.flag = cflag;
  cp.batch = batch;
  cp.max_pages = max_pages_per_seq;
  cp.q_len = q_len;
  cp.prefix_len = prefix_len;
  cudaError_t e = mla::launch_cascade_prep(cp, s);
  if (e != cudaSuccess) return cuda_fail(e, "cascade prep launch");
  // prefix pass: every query row of the batch, one sequence of prefix_len tokens (sequence 0's pages)
  void* wpre = ws + o_pre;
  void* wsuf = ws + o_suf;
  size_t cap = ws_pre;
  if ((st = plan_impl(sl_pre, block_table, num_pages, 1, max_pages_per_seq, 1, rows, kv_dtype, 0, wpre, &cap, nullptr,
                      stream, true)) != MLA_OK)
    return st;
  if ((st = run_impl(q, kv_cache, num_pages, kv_dtype, block_table, sl_pre, ws + o_out1,
                     reinterpret_cast<float*>(ws + o_lse1), 1, max_pages_per_seq, 1, rows, scale, wpre, ws_pre,
                     MLA_PHASE_ATTEND | MLA_PHASE_COMBINE, stream, true)) != MLA_OK)
    return st;
  // suffix pass: each sequence's pages from prefix_len / 64 on (the block-table rows keep their stride)
  const int32_t* bt_suf = block_table + prefix_len / mla::kPage;
  cap = ws_suf;
  if ((st = plan_impl(sl_suf, bt_suf, num_pages, batch, max_pages_per_seq, q_len, heads, kv_dtype, 0, wsuf, &cap,
                      nullptr, stream, false)) != MLA_OK)
    return st;
  if ((st = run_impl(q, kv_cache, num_pages, kv_dtype, bt_suf, sl_suf, ws + o_out2,
                     reinterpret_cast<float*>(ws + o_lse2), batch, max_pages_per_seq, q_len, heads, scale, wsuf,
                     ws_suf, MLA_PHASE_ATTEND | MLA_PHASE_COMBINE, stream, false)) != MLA_OK)
    return st;
  mla::MergeParams mp;
  mp.out_a = reinterpret_cast<const uint16_t*>(ws + o_out1);
  mp.lse_a = reinterpret_cast<const float*>(ws + o_lse1);
  mp.out_b = reinterpret_cast<const uint16_t*>(ws + o_out2);
  mp.lse_b = reinterpret_cast<const float*>(ws + o_lse2);
  mp.out = static_cast<uint16_t*>(out);
  mp.lse = lse;
  mp.rows = rows;
  mp.flag_prefix = reinterpret_cast<int32_t*>(wpre);
  mp.flag_suffix = reinterpret_cast<const int32_t*>(wsuf);
  mp.flag_prep = cflag;
  if ((e = mla::launch_merge(mp, s)) != cudaSuccess) return cuda_fail(e, "merge kernel launch");
  return MLA_OK;
}

int mla_cache_append(const void* kv_new, void* kv_cache, int64_t num_pages, int kv_dtype, const int32_t* block_table,
                     const int32_t* seqlens, int batch, int max_pages_per_seq, int q_len, int32_t* flag,
                     void* stream) {
  g_last_error.clear();
  int st = check_shape(batch, max_pages_per_seq, q_len, 1, kv_dtype);
  if (st != MLA_OK) return st;
  if (num_pages < 1 || num_pages > 0x7FFFFFFFll)
    return fail(MLA_ERR_INVALID_ARG, "num_pages must be in [1, 2^31-1] (got %lld)", (long long)num_pages);
  if (batch == 0) return MLA_OK;
  const struct {
    const void* p;
    const char* name;
    size_t align;
  } ptrs[] = {{kv_new, "kv_new", 16}, {kv_cache, "kv_cache", 16}, {block_table, "block_table", 4},
              {seqlens, "seqlens", 4}};
  for (const auto& x : ptrs) {
    if (!x.p) return fail(MLA_ERR_INVALID_ARG, "%s is NULL", x.name);
    if (!aligned(x.p, x.align)) return fail(MLA_ERR_INVALID_ARG, "%s must be %zu-byte aligned", x.name, x.align);
  }
  if (flag && !aligned(flag, 4)) return fail(MLA_ERR_INVALID_ARG, "flag must be 4-byte aligned");
  for (const auto& x : ptrs)
    if ((st = check_device_ptr(x.p, x.name)) != MLA_OK) return st;
  if (flag && (st = check_device_ptr(flag, "flag")) != MLA_OK) return st;
  mla::AppendParams p;
  p.src = static_cast<const uint16_t*>(kv_new);
  p.cache = kv_cache;
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.flag = flag;
  p.num_pages = num_pages;
  p.batch = batch;
  p.max_pages = max_pages_per_seq;
  p.q_len = q_len;
  p.fp8 = kv_dtype == MLA_KV_FP8_E4M3 ? 1 : 0;
  const cudaError_t e = mla::launch_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  return MLA_OK;
}

namespace {

// Shared argument checks and tensor maps of the two projections.
int projection(bool absorb, const void* x, const void* w, void* out, int n_tokens, int heads, int32_t* flag,
               void* stream) {
  g_last_error.clear();
  if (n_tokens < 0 || n_tokens > (1 << 20))
    return fail(MLA_ERR_UNSUPPORTED, "n_tokens must be in [0, 2^20] (got %d)", n_tokens);
  if (heads < 1 || heads > 128) return fail(MLA_ERR_UNSUPPORTED, "heads must be in [1, 128] (got %d)", heads);
  if (n_tokens == 0) return MLA_OK;
  const char* xname = absorb ? "q" : "o";
  const char* wname = absorb ? "w_uk" : "w_uv";
  const char* oname = absorb ? "q_out" : "y";
  const struct {
    const void* p;
    const char* name;
  } ptrs[] = {{x, xname}, {w, wname}, {out, oname}};
  int st;
  for (const auto& a : ptrs) {
    if (!a.p) return fail(MLA_ERR_INVALID_ARG, "%s is NULL", a.name);
    if (!aligned(a.p, 16)) return fail(MLA_ERR_INVALID_ARG, "%s must be 16-byte aligned", a.name);
  }
  if (flag && !aligned(flag, 4)) return fail(MLA_ERR_INVALID_ARG, "flag must be 4-byte aligned");
  for (const auto& a : ptrs)
    if ((st = check_device_ptr(a.p, a.name)) != MLA_OK) return st;
  if (flag && (st = check_device_ptr(flag, "flag")) != MLA_OK) return st;
  DeviceInfo d;
  if ((st = device_info(&d)) != MLA_OK) return st;
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  int dev = 0;
  cudaGetDevice(&dev);
  const cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap tm_a, tm_b;
  // activations [n_tokens][heads][width]: boxes of 64 columns x 1 head x 128 tokens
  const cuuint64_t width = absorb ? 192 : 512;
  const MapKey ka{dev, absorb ? 8 : 10, x, static_cast<unsigned long long>(n_tokens), static_cast<unsigned long long>(heads)};
  if (!map_lookup(ka, &tm_a)) {
    const cuuint64_t dims[3] = {width, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(n_tokens)};
    const cuuint64_t strides[2] = {width * 2, width * 2 * static_cast<cuuint64_t>(heads)};
    const cuuint32_t box[3] = {64, 1, 128};
    CUresult r = enc(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed (%d)", xname, static_cast<int>(r));
    map_store(ka, tm_a);
  }
  // weights [heads][128][512]: absorb boxes 64 columns x 64 rows, project 64 columns x 32 rows
  const MapKey kb{dev, absorb ? 9 : 11, w, static_cast<unsigned long long>(heads), 0};
  if (!map_lookup(kb, &tm_b)) {
    const cuuint64_t dims[3] = {512, 128, static_cast<cuuint64_t>(heads)};
    const cuuint64_t strides[2] = {512 * 2, 512 * 2 * 128};
    const cuuint32_t box[3] = {64, absorb ? 64u : 32u, 1};
    CUresult r = enc(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed (%d)", wname, static_cast<int>(r));
    map_store(kb, tm_b);
  }
  mla::ProjParams p;
  p.in = static_cast<const uint16_t*>(x);
  p.out = static_cast<uint16_t*>(out);
  p.flag = flag;
  p.n_tokens = n_tokens;
  p.heads = heads;
  p.out_row = absorb ? mla::kDqk : 128;
  p.timeout_ns = g_timeout_ns;
  const cudaError_t e = mla::launch_proj(absorb, tm_a, tm_b, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, absorb ? "absorb kernel launch" : "projection kernel launch");
  return MLA_OK;
}

}  // namespace

int mla_absorb_q(const void* q, const void* w_uk, void* q_out, int n_tokens, int heads, int32_t* flag,
                 void* stream) {
  return projection(true, q, w_uk, q_out, n_tokens, heads, flag, stream);
}

int mla_project_out(const void* o, const void* w_uv, void* y, int n_tokens, int heads, int32_t* flag,
                    void* stream) {
  return projection(false, o, w_uv, y, n_tokens, heads, flag, stream);
}

int mla_read_device_flag(const void* workspace, int* flag, void* stream) {
  g_last_error.clear();
  if (!workspace || !flag) return fail(MLA_ERR_INVALID_ARG, "workspace and flag must be non-NULL");
  int v = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device flag");
  *flag = v;
  if (v != 0) return fail(MLA_ERR_DEVICE_FLAG, "device flag 0x%x%s%s%s", v, (v & 1) ? " timeout" : "",
                          (v & 2) ? " bad-seqlen" : "", (v & 4) ? " bad-page" : "");
  return MLA_OK;
}

}  // extern "C"
