// K2: LSE-weighted merge of split-KV partials.
//
// A sequence cut into s > 1 pieces by the planner has, per query row, s fp32
// partials (O_i normalised by its own softmax denominator, lse_i). With
// lse* = log sum_i exp(lse_i), the exact result is
//     out = sum_i exp(lse_i - lse*) O_i,       lse = lse*.
//
// Work decomposition: the planner lists the sequences with splits != 1 and
// the number of work items each needs (combine_items). A persistent grid of a
// few CTAs per SM walks the work items; an item is 8 warps, and a task (one
// query row x one 128-column chunk, lane = 4 columns) takes combine_warps(s)
// of them, each summing a contiguous share of the pieces with all its partial
// loads in flight at once; shares are added in shared memory. Sequences held
// by one cluster were finished by K1 and are not listed; sequences the planner
// rejected (bad length) are listed with s = 0 and get NaN rows.
//
// Placement. The work items' partial loads bound the kernel: about 28 KB/us of
// L2 reads per SM were measured, whatever the item count. CTAs start on SMs as
// the decode kernel's clusters finish, a few per freed SM, so when a step has
// few items (at most two per SM: one sequence of <= 74 query rows gives at
// most rows * 4) the first SMs to free up took all of them, four per SM, while
// the rest sat idle. Such launches use the "spread" instance: one CTA per item and
// enough (unused) dynamic shared memory that at most two CTAs fit on an SM.
#include <cmath>
#include <mutex>

#include <cuda_bf16.h>

#include "mla_common.cuh"
#include "mla_launch.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kCombineThreads = kCombineWarps * 32;
constexpr int kUnroll = 9;   // partial rows in flight per lane (s <= 72 pieces: one round)

// 4-byte global -> shared copy that holds no register while in flight.
__device__ __forceinline__ void cp_async_4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

#ifdef MLA_TRACE
#define MLA_K2_EXIT()                                                                                 \
  do {                                                                                                \
    if (threadIdx.x == 0 && p.trace != nullptr)                                                       \
      atomicMax(reinterpret_cast<unsigned long long*>(p.trace) + kTraceStepBase + 3, globaltimer_ns()); \
  } while (0)
#else
#define MLA_K2_EXIT() \
  do {                \
  } while (0)
#endif

// Dynamic shared memory of a spread launch: 12 KB static + this + 1 KB reserved
// per CTA lets two CTAs, not three, share an SM's 228 KB.
constexpr int kSpreadSmemBytes = 80 * 1024;

// kSpread only selects the instance (and so its launch attributes); the code is the same.
template <bool kSpread>
__global__ void __launch_bounds__(kCombineThreads, 4) mla_combine_kernel(const CombineParams p) {
  __shared__ float wgt[kCombineWarps][kCombineMaxSplits];   // per warp: exp(lse_i - max) of its task
  __shared__ float4 red[kCombineWarps][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#ifdef MLA_TRACE
  unsigned long long* tr = reinterpret_cast<unsigned long long*>(p.trace);
  if (tid == 0 && tr != nullptr) atomicMin(tr + kTraceStepBase + 2, globaltimer_ns());
#endif

  pdl_wait();  // partials and plan of the decode kernel
#ifdef MLA_TRACE
  if (tid == 0 && tr != nullptr) atomicMin(tr + kTraceStepBase + 4, globaltimer_ns());
#endif

  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  const char* ws = reinterpret_cast<const char*>(p.ws);
  const int32_t* seq = reinterpret_cast<const int32_t*>(ws + w.seq_off);
  const int32_t* list = reinterpret_cast<const int32_t*>(ws + w.list_off);
  const int32_t* vcp = reinterpret_cast<const int32_t*>(ws + w.vcp_off);
  const float* plse = reinterpret_cast<const float*>(ws + w.plse_off);
  const float* po = reinterpret_cast<const float*>(ws + w.po_off);
  const int listed = p.ws[kHdrListed];
  const int items = p.ws[kHdrCombineCtas];
  const size_t piece_stride = static_cast<size_t>(p.row_tiles) * kRowsPerTile;   // rows between pieces

  for (int v = blockIdx.x; v < items; v += gridDim.x) {
    // listed sequence k: the first whose inclusive item prefix exceeds v
    int lo = 0, hi = listed - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (vcp[mid] > v) hi = mid; else lo = mid + 1;
    }
    const int k = lo;
    const int b = list[k];
    const int32_t* sq = seq + static_cast<size_t>(b) * kSeqWords;
    const int s = sq[kSeqSplits];
    const int slot = sq[kSeqSlot];
    const int nw = combine_warps(s);
    const int task = (v - (k > 0 ? vcp[k - 1] : 0)) * (kCombineWarps / nw) + warp / nw;
    const int sub = warp % nw;
    const bool valid = task < p.rows * 4;
    const int r = task >> 2, chunk = task & 3;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float mx = -INFINITY, den = 0.f;
    if (valid && s > 0) {
      const int rt = r / p.tile_rows, rr = r % p.tile_rows;
      const size_t idx0 = (static_cast<size_t>(slot) * p.row_tiles + rt) * kRowsPerTile + rr;
      const float* src = po + idx0 * kDv + chunk * 128 + lane * 4;
      const int per = (s + nw - 1) / nw;
      const int j0 = min(s, sub * per), j1 = min(s, j0 + per);
      // the first partial rows of this warp's share go out before the weights are known
      float4 o[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (j0 + u < j1) o[u] = __ldg(reinterpret_cast<const float4*>(src + (j0 + u) * piece_stride * kDv));
      // All of the task's lse_i go out at once, parked in this lane's weight slots (a
      // loop of plain loads would wait for each one before the next: one L2 round trip
      // per 32 pieces).
      for (int j = lane; j < s; j += 32) cp_async_4(&wgt[warp][j], plse + idx0 + j * piece_stride);
      cp_async_wait_all();
      for (int j = lane; j < s; j += 32) mx = fmaxf(mx, wgt[warp][j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      for (int j = lane; j < s; j += 32) {
        const float ls = wgt[warp][j];
        const float e = (ls == -INFINITY) ? 0.f : __expf(ls - mx);   // a piece in which this row saw no token
        wgt[warp][j] = e;
        den += e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
      __syncwarp();
      for (int j = j0; j < j1; j += kUnroll) {
        if (j > j0) {
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (j + u < j1) o[u] = __ldg(reinterpret_cast<const float4*>(src + (j + u) * piece_stride * kDv));
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          if (j + u < j1) {
            const float e = wgt[warp][j + u];
            acc.x += e * o[u].x;
            acc.y += e * o[u].y;
            acc.z += e * o[u].z;
            acc.w += e * o[u].w;
          }
        }
      }
    }
    if (nw > 1) {   // add the shares of the task's warps (uniform over the CTA: one sequence per item)
      red[warp][lane] = acc;
      __syncthreads();
      if (sub == 0) {
        for (int q = 1; q < nw; ++q) {
          const float4 t = red[warp + q][lane];
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        }
      }
    }
    if (valid && sub == 0) {
      uint2* dst = reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(b) * p.rows + r) * kDv + chunk * 128) + lane;
      if (s == 0) {
        *dst = make_uint2(0x7FC07FC0u, 0x7FC07FC0u);
        if (chunk == 0 && lane == 0) p.lse[static_cast<size_t>(b) * p.rows + r] = __int_as_float(0x7FC00000);
      } else {
        const float inv = den > 0.f ? 1.f / den : 0.f;
        *dst = make_uint2(pack2(acc.x * inv, acc.y * inv), pack2(acc.z * inv, acc.w * inv));
        if (chunk == 0 && lane == 0)
          p.lse[static_cast<size_t>(b) * p.rows + r] = den > 0.f ? mx + logf(den) : -INFINITY;
      }
    }
    __syncthreads();   // wgt / red are reused by the next item
  }
  MLA_K2_EXIT();
}

// SM count of the current device, and (once per device) the spread instance's
// shared-memory attributes.
cudaError_t combine_device(int* sms) {
  static std::mutex mu;
  static int sm_count[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (sm_count[dev] == 0) {
    int n = 0;
    if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(mla_combine_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kSpreadSmemBytes)) != cudaSuccess)
      return e;
    // the whole unified memory as shared memory, so that two spread CTAs fit
    if ((e = cudaFuncSetAttribute(mla_combine_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    sm_count[dev] = n;
  }
  *sms = sm_count[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  if (p.c_max > kCombineMaxSplits || p.grid < 1) return cudaErrorInvalidValue;
  int sms = 0;
  const cudaError_t e = combine_device(&sms);
  if (e != cudaSuccess) return e;
  // A grid of at most two CTAs per SM is a one-CTA-per-item launch: spread it.
  const bool spread = p.grid <= 2 * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid), 1, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
  cfg.dynamicSmemBytes = spread ? kSpreadSmemBytes : 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return spread ? cudaLaunchKernelEx(&cfg, mla_combine_kernel<true>, p)
                : cudaLaunchKernelEx(&cfg, mla_combine_kernel<false>, p);
}

}  // namespace mla
