// K2: LSE-weighted merge of split-KV partials.
//
// A sequence cut into s > 1 pieces by the planner has, per query row, s fp32
// partials (O_i normalised by its own softmax denominator, lse_i). With
// lse* = log sum_i exp(lse_i), the exact result is
//     out = sum_i exp(lse_i - lse*) O_i,       lse = lse*.
// One CTA per (sequence, query row, 128-column chunk): the weights are formed
// once in shared memory, then 8 groups of 32 threads each sum every 8th piece
// (4 columns per thread, all loads independent) and a shared-memory reduction
// finishes the row. Sequences held by one cluster were finished by K1 and are
// skipped; sequences the planner rejected (bad length) get NaN rows.
#include <cmath>

#include <cuda_bf16.h>

#include "mla_common.cuh"
#include "mla_launch.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kChunks = kDv / 128;       // 4 column chunks of 128
constexpr int kGroups = 8;               // piece groups per CTA
constexpr int kMaxPieces = 1024;         // >= clusters per row tile

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

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const CombineParams p) {
  __shared__ float wgt[kMaxPieces];
  __shared__ float4 red[kGroups][32];
  __shared__ float s_max, s_den;

  const long long bid = blockIdx.x;
  const int chunk = static_cast<int>(bid % kChunks);
  const long long br = bid / kChunks;
  const int b = static_cast<int>(br / p.rows);
  const int rg = static_cast<int>(br % p.rows);
  const int tid = threadIdx.x, cg = tid & 31, sg = tid >> 5;
#ifdef MLA_TRACE
  unsigned long long* tr = reinterpret_cast<unsigned long long*>(p.trace);
  if (tid == 0 && tr != nullptr) atomicMin(tr + kTraceStepBase + 2, globaltimer_ns());
#endif

  pdl_wait();  // partials and plan of the decode kernel
#ifdef MLA_TRACE
  if (tid == 0 && tr != nullptr) atomicMin(tr + kTraceStepBase + 4, globaltimer_ns());
#endif

  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  const int32_t* sq = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.seq_off) +
                      static_cast<size_t>(b) * kSeqWords;
  const int splits = sq[kSeqSplits];
  if (splits == 1) {
    MLA_K2_EXIT();
    return;
  }
  uint16_t* orow = p.out + static_cast<size_t>(br) * kDv + chunk * 128;
  if (splits == 0) {
    if (tid < 32) reinterpret_cast<uint2*>(orow)[tid] = make_uint2(0x7FC07FC0u, 0x7FC07FC0u);
    if (tid == 0 && chunk == 0) p.lse[br] = __int_as_float(0x7FC00000);
    MLA_K2_EXIT();
    return;
  }
  const float* plse = reinterpret_cast<const float*>(reinterpret_cast<const char*>(p.ws) + w.plse_off);
  const float* po = reinterpret_cast<const float*>(reinterpret_cast<const char*>(p.ws) + w.po_off);
  const int r = rg / p.tile_rows, row = rg % p.tile_rows;
  const size_t idx0 = (static_cast<size_t>(sq[kSeqSlot]) * p.row_tiles + r) * kRowsPerTile + row;
  const size_t idx_stride = static_cast<size_t>(p.row_tiles) * kRowsPerTile;

  for (int s = tid; s < splits; s += kCombineThreads) wgt[s] = plse[idx0 + s * idx_stride];
  __syncthreads();
  if (sg == 0) {
    float mx = -INFINITY;
    for (int s = cg; s < splits; s += 32) mx = fmaxf(mx, wgt[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.f;
    for (int s = cg; s < splits; s += 32) {
      const float ls = wgt[s];
      const float e = (ls == -INFINITY) ? 0.f : __expf(ls - mx);   // a piece in which this row saw no token
      wgt[s] = e;
      den += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (cg == 0) {
      s_max = mx;
      s_den = den;
    }
  }
  __syncthreads();

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* src = po + idx0 * kDv + chunk * 128 + cg * 4;
#pragma unroll 4
  for (int s = sg; s < splits; s += kGroups) {
    const float e = wgt[s];
    const float4 o = *reinterpret_cast<const float4*>(src + static_cast<size_t>(s) * idx_stride * kDv);
    acc.x += e * o.x;
    acc.y += e * o.y;
    acc.z += e * o.z;
    acc.w += e * o.w;
  }
  red[sg][cg] = acc;
  __syncthreads();
  if (sg == 0) {
    float4 t = red[0][cg];
#pragma unroll
    for (int k = 1; k < kGroups; ++k) {
      const float4 u = red[k][cg];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
    }
    const float inv = 1.f / s_den;
    reinterpret_cast<uint2*>(orow)[cg] = make_uint2(pack2(t.x * inv, t.y * inv), pack2(t.z * inv, t.w * inv));
    if (cg == 0 && chunk == 0) p.lse[br] = s_max + logf(s_den);
  }
  MLA_K2_EXIT();
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const long long blocks = static_cast<long long>(p.batch) * p.rows * kChunks;
  if (blocks == 0) return cudaSuccess;
  if (p.c_max > kMaxPieces) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_combine_kernel, p);
}

}  // namespace mla
