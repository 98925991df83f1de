// Prefix-shared (cascade) decode: the kernels around the two decode passes.
//
// The pages describe multi-turn agentic serving in which sequences share the
// KV pages of a common prefix (zubnet.ai, "LightSeek TokenSpeed 580 TPS ...
// B200", second paragraph: hybrid prefix caching; 24-ai.news "TokenSpeed ...
// 580 token/s", optimisations list: prefix caching, KV hit rate above 90%).
// A cascade step splits each row's visible tokens into the shared prefix
// (tokens 0 .. P-1, pages common to every sequence of the call, all visible
// to every query) and the sequence's own suffix (P .. L_b - 1, causal among
// the q_len new tokens). The prefix pass attends the union of the batch's
// query rows to the prefix as ONE sequence, so a 128-row tile holds the rows
// of several sequences and loads each prefix page once for all of them; the
// suffix pass is an ordinary decode over each sequence's remaining pages.
// The two partial results are merged by their log-sum-exp weights:
//   lse = log(e^lse_a + e^lse_b),  out = e^(lse_a - lse) out_a + e^(lse_b - lse) out_b.
//
//   mla_cascade_prep_kernel : suffix lengths L_b - P, the prefix length as a
//                             one-sequence batch, and a check that every
//                             sequence's first P/64 block-table entries equal
//                             sequence 0's (the pages are really shared)
//   mla_merge_kernel        : the merge, one warp per query row
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "mla_common.cuh"
#include "mla_launch.h"

namespace mla {

namespace {

__global__ void __launch_bounds__(256) mla_cascade_prep_kernel(const CascadeParams p) {
  const int prefix_pages = p.prefix_len / kPage;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  int bad = 0;
  // every sequence's first prefix_pages block-table entries must be sequence 0's
  for (long long idx = tid; idx < static_cast<long long>(p.batch) * prefix_pages; idx += stride) {
    const long long b = idx / prefix_pages, i = idx % prefix_pages;
    if (b > 0 && p.block_table[b * p.max_pages + i] != p.block_table[i]) bad |= kFlagBadPrefix;
  }
  for (long long b = tid; b < p.batch; b += stride) {
    const int L = p.seqlens[b];
    const bool ok = L >= p.prefix_len + p.q_len && L <= p.max_pages * kPage;
    p.seqlens_suffix[b] = ok ? L - p.prefix_len : 0;   // 0 < q_len: the suffix pass flags it and writes NaN rows
    if (!ok) bad |= kFlagBadSeqlen;
  }
  if (tid == 0) p.seqlen_prefix[0] = p.prefix_len;
  if (bad) atomicOr(p.flag, bad);
}

__global__ void __launch_bounds__(256) mla_cascade_clear_kernel(const CascadeParams p) {
  if (threadIdx.x == 0) p.flag[0] = 0;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One warp per query row: lane l takes columns 16l .. 16l + 15 (two 16-byte
// chunks of each input). The flag words of both passes and of the prep are
// folded into the prefix workspace's flag word (the one the caller reads).
__global__ void __launch_bounds__(256) mla_merge_kernel(const MergeParams p) {
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const int f = p.flag_suffix[0] | p.flag_prep[0];
    if (f) atomicOr(p.flag_prefix, f);
  }
  if (r >= p.rows) return;
  const float la = p.lse_a[r], lb = p.lse_b[r];
  float m = fmaxf(la, lb);
  float wa, wb;
  if (isnan(la) || isnan(lb)) {        // an invalid sequence: NaN rows, as the decode writes them
    wa = wb = __int_as_float(0x7FC00000);
    m = wa;
  } else {
    if (m == -INFINITY) m = 0.f;
    wa = la == -INFINITY ? 0.f : expf(la - m);
    wb = lb == -INFINITY ? 0.f : expf(lb - m);
  }
  const float den = wa + wb;
  const float inv = 1.f / den;
  const uint4* a = reinterpret_cast<const uint4*>(p.out_a + r * kDv) + 2 * lane;
  const uint4* b = reinterpret_cast<const uint4*>(p.out_b + r * kDv) + 2 * lane;
  uint4* o = reinterpret_cast<uint4*>(p.out + r * kDv) + 2 * lane;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint4 x = a[k], y = b[k];
    const uint32_t xa[4] = {x.x, x.y, x.z, x.w}, yb[4] = {y.x, y.y, y.z, y.w};
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = pack((wa * bf16_lo(xa[i]) + wb * bf16_lo(yb[i])) * inv, (wa * bf16_hi(xa[i]) + wb * bf16_hi(yb[i])) * inv);
    o[k] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (lane == 0) p.lse[r] = m + logf(den);
}

}  // namespace

cudaError_t launch_cascade_prep(const CascadeParams& p, cudaStream_t stream) {
  mla_cascade_clear_kernel<<<1, 32, 0, stream>>>(p);
  const long long work = static_cast<long long>(p.batch) * (p.prefix_len / kPage > 1 ? p.prefix_len / kPage : 1);
  long long blocks = (work + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 592) blocks = 592;
  mla_cascade_prep_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  if (p.rows == 0) return cudaSuccess;
  mla_merge_kernel<<<static_cast<unsigned>((p.rows + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
