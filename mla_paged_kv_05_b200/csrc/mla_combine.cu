// K2: LSE-weighted merge of split-KV partials.
//
// A sequence cut into s > 1 pieces by the planner has, per query row, s fp32
// partials (O_i normalised by its own softmax denominator, lse_i). With
// lse* = log sum_i exp(lse_i), the exact result is
//     out = sum_i exp(lse_i - lse*) O_i,       lse = lse*.
// One warp per (sequence, query row); each lane owns 16 of the 512 columns.
// Sequences held by a single cluster were finished by K1 and are skipped;
// sequences the planner rejected (bad length) get NaN rows.
#include <cmath>

#include <cuda_bf16.h>

#include "mla_common.cuh"
#include "mla_launch.h"

namespace mla {

namespace {

constexpr int kCombineWarps = 8;

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kCombineWarps * 32) mla_combine_kernel(const CombineParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * kCombineWarps + warp;
  if (gw >= static_cast<long long>(p.batch) * p.rows) return;
  const int b = static_cast<int>(gw / p.rows);
  const int rg = static_cast<int>(gw % p.rows);
  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  const int32_t* sq = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.seq_off) +
                      static_cast<size_t>(b) * kSeqWords;
  const int splits = sq[kSeqSplits];
  if (splits == 1) return;
  uint16_t* orow = p.out + static_cast<size_t>(gw) * kDv + lane * 16;
  if (splits == 0) {
    const uint32_t nan2 = 0x7FC07FC0u;
    reinterpret_cast<uint4*>(orow)[0] = make_uint4(nan2, nan2, nan2, nan2);
    reinterpret_cast<uint4*>(orow)[1] = make_uint4(nan2, nan2, nan2, nan2);
    if (lane == 0) p.lse[gw] = __int_as_float(0x7FC00000);
    return;
  }
  const float* plse = reinterpret_cast<const float*>(reinterpret_cast<const char*>(p.ws) + w.plse_off);
  const float* po = reinterpret_cast<const float*>(reinterpret_cast<const char*>(p.ws) + w.po_off);
  const int r = rg / kRowsPerTile, row = rg % kRowsPerTile;
  const int slot0 = sq[kSeqSlot];

  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const size_t idx = (static_cast<size_t>(slot0 + s) * p.row_tiles + r) * kRowsPerTile + row;
    mx = fmaxf(mx, plse[idx]);
  }
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float den = 0.f;
  for (int s = 0; s < splits; ++s) {
    const size_t idx = (static_cast<size_t>(slot0 + s) * p.row_tiles + r) * kRowsPerTile + row;
    const float ls = plse[idx];
    if (ls == -INFINITY) continue;     // a piece in which this row saw no token
    const float wgt = __expf(ls - mx);
    den += wgt;
    const float4* src = reinterpret_cast<const float4*>(po + idx * kDv + lane * 16);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 o = src[v];
      acc[4 * v] += wgt * o.x;
      acc[4 * v + 1] += wgt * o.y;
      acc[4 * v + 2] += wgt * o.z;
      acc[4 * v + 3] += wgt * o.w;
    }
  }
  const float inv = 1.f / den;
  uint4* dst = reinterpret_cast<uint4*>(orow);
  dst[0] = make_uint4(pack2(acc[0] * inv, acc[1] * inv), pack2(acc[2] * inv, acc[3] * inv),
                      pack2(acc[4] * inv, acc[5] * inv), pack2(acc[6] * inv, acc[7] * inv));
  dst[1] = make_uint4(pack2(acc[8] * inv, acc[9] * inv), pack2(acc[10] * inv, acc[11] * inv),
                      pack2(acc[12] * inv, acc[13] * inv), pack2(acc[14] * inv, acc[15] * inv));
  if (lane == 0) p.lse[gw] = mx + logf(den);
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const long long warps = static_cast<long long>(p.batch) * p.rows;
  if (warps == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((warps + kCombineWarps - 1) / kCombineWarps);
  mla_combine_kernel<<<blocks, kCombineWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
