// Latent-cache append: the write that precedes a decode step.
//
// The q_len new tokens of each sequence (the last q_len positions, already
// counted in seqlens: L_b - q_len .. L_b - 1) get their 576-wide latent rows
// written into their cache pages through the block table - KV pages reached
// by index indirection instead of copies (zubnet.ai "LightSeek TokenSpeed 580
// TPS ... B200", second paragraph). A bf16 cache takes the row as it is. An
// fp8-e4m3 cache takes codes and one fp32 scale per token: sigma = amax|x|/448
// (1 for an all-zero row) and code = e4m3(x / sigma), nearest-even and
// saturated to +-448 (OCP 8-bit floating point, E4M3). The pages give no
// quantisation rule; this is the library's reading, the same one its decode
// kernel's fp8 path assumes. Both divisions are IEEE fp32 (round to nearest),
// so the codes are a deterministic function of the row. (A reciprocal with an
// FMA-corrected quotient and an exactness guard was tried in place of the
// per-element division: exact, but slower on B200.)
//
// One warp per new row: 72 chunks of 16 bytes (8 bf16), three per lane, read
// and written with coalesced 16-byte (bf16) or 8-byte (fp8 codes) accesses.
// The work is bound by HBM: 1,152 bytes read and 1,152 (bf16) or 580 (fp8)
// bytes written per row, plus the block-table entry.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/mla_decode.h"
#include "mla_common.cuh"
#include "mla_launch.h"

namespace mla {

namespace {

constexpr int kAppendWarps = 8;                // rows per CTA
constexpr int kChunks = kDqk / 8;              // 16-byte chunks of a bf16 row (72)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 values -> two e4m3 codes (first value in the low byte), nearest-even, saturated.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float first, float second) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
  return r;
}

__global__ void __launch_bounds__(kAppendWarps * 32) mla_append_kernel(const AppendParams p) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kAppendWarps + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(p.batch) * p.q_len) return;
  const int b = static_cast<int>(row / p.q_len), t = static_cast<int>(row % p.q_len);
  const int L = p.seqlens[b];
  if (L < p.q_len || L > p.max_pages * kPage) {
    if (lane == 0 && p.flag != nullptr) atomicOr(p.flag, kFlagBadSeqlen);
    return;
  }
  const int j = L - p.q_len + t;
  const int page = p.block_table[static_cast<size_t>(b) * p.max_pages + j / kPage];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0 && p.flag != nullptr) atomicOr(p.flag, kFlagBadPage);
    return;
  }
  const int slot = j % kPage;
  const uint4* src = reinterpret_cast<const uint4*>(p.src) + row * kChunks;
  uint4 v[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int c = lane + 32 * k;
    v[k] = c < kChunks ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (!p.fp8) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.cache) +
                                          (static_cast<size_t>(page) * kPage + slot) * kDqk * 2);
#pragma unroll
    for (int k = 0; k < 3; ++k)
      if (lane + 32 * k < kChunks) dst[lane + 32 * k] = v[k];
    return;
  }
  // fp8: the row's largest magnitude, then codes of x / sigma
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sigma = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* pg = static_cast<uint8_t*>(p.cache) + static_cast<size_t>(page) * kFp8PageBytes;
  uint2* dst = reinterpret_cast<uint2*>(pg + static_cast<size_t>(slot) * kDqk);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int c = lane + 32 * k;
    if (c >= kChunks) continue;
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q[i] = e4m3x2_from_f32(__fdiv_rn(bf16_lo(w[i]), sigma), __fdiv_rn(bf16_hi(w[i]), sigma));
    dst[c] = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
  }
  if (lane == 0) reinterpret_cast<float*>(pg + kPage * kDqk)[slot] = sigma;
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.batch) * p.q_len;
  if (rows == 0) return cudaSuccess;
  const long long grid = (rows + kAppendWarps - 1) / kAppendWarps;
  mla_append_kernel<<<static_cast<unsigned>(grid), kAppendWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
