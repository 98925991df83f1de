// Absorbed-MLA projections around the decode attention, on the tensor cores.
//
// The pages name an MLA decode kernel (evermx.com, "TokenSpeed: speed-of-light
// LLM inference engine for agentic workloads", section "Pluggable Kernel
// Registry") but not its algebra. In the absorbed form the decode attention
// reads one shared 512-wide latent per token; the per-head up-projections
// W_UK[h], W_UV[h] (128 x 512 each) move to the query and the output:
//
//   absorb : q~[n][h] = [W_UK[h]^T q[n][h][0:128] | q[n][h][128:192]]   (576 wide)
//   project: y[n][h]  = W_UV[h] o[n][h]                                  (128 wide)
//
// for the n_tokens = batch * q_len query tokens of a step. Each is a batch of
// per-head GEMMs whose token count is small and whose weights (16 MB per
// projection at 128 heads) dominate the bytes, so HBM bounds them. A CTA
// takes one head, one tile of up to 128 tokens and a slice of the head's
// output; the tokens are the M = 128
// rows of tcgen05.mma kind::f16 (rows past n_tokens are TMA zero fill, read
// from no memory), fp32 accumulators in tensor memory, operands staged by TMA
// in 128-byte swizzled boxes:
//   absorb : A = q nope [128 tokens x 128] K-major; B = 128 of W_UK[h]'s 512
//            columns (MN-major: the output columns are contiguous); D = 128 x
//            128. Four CTAs per head.
//   project: A = o [128 tokens x 512] K-major; B = 32 of W_UV[h]'s 128 rows
//            (K-major); D = 128 x 32; the eight 64-wide K chunks stream through
//            a four-stage ring. Four CTAs per head.
// Roles: warp 0 lane 0 issues TMA, warp 1 lane 0 issues MMAs (warp 1 owns the
// TMEM allocation), then all four warps read their 32 TMEM lanes (token rows)
// and store bf16 rows. Every wait is bounded; a wait that runs out sets
// MLA_FLAG_TIMEOUT in the caller's flag word (if any) and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla_decode.h"
#include "mla_common.cuh"
#include "mla_launch.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kProjThreads = 128;
constexpr int kBoxBytes = 64 * 128;   // 64 rows x 64 bf16 (128 bytes), 128B swizzle
constexpr unsigned long long kProjDrainNs = 200ull * 1000 * 1000;

// Each head's output is split over kSplits CTAs (more CTAs in flight than heads).
template <bool kAbsorb>
struct ProjCfg;
template <>
struct ProjCfg<true> {                 // absorb: a CTA takes 128 of the 512 latent columns
  static constexpr int kSplits = 4;
  static constexpr int kChunks = 2;    // K = 128 in chunks of 64
  static constexpr int kStages = 2;
  static constexpr int kABytes = 128 * 128;        // 128 token rows x 64 K
  static constexpr int kBBytes = 2 * kBoxBytes;    // 64 K rows x 128 N, as 2 boxes of 64 N
  static constexpr uint32_t kTmemCols = 128;
  static constexpr int kN = 128;
};
template <>
struct ProjCfg<false> {                // project: a CTA takes 32 of the 128 output dimensions
  static constexpr int kSplits = 4;
  static constexpr int kChunks = 8;    // K = 512 in chunks of 64
  static constexpr int kStages = 4;
  static constexpr int kABytes = 128 * 128;        // 128 token rows x 64 K
  static constexpr int kBBytes = 32 * 128;         // 32 N rows x 64 K
  static constexpr uint32_t kTmemCols = 32;
  static constexpr int kN = 32;
};

template <bool kAbsorb>
constexpr int proj_smem_bytes() {
  return ProjCfg<kAbsorb>::kStages * (ProjCfg<kAbsorb>::kABytes + ProjCfg<kAbsorb>::kBBytes) + 1024 + 1024;
}

template <int kStages>
struct ProjBars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <bool kAbsorb>
__global__ void __launch_bounds__(kProjThreads, 1)
    mla_proj_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const ProjParams p) {
  using C = ProjCfg<kAbsorb>;
  constexpr int kStage = C::kABytes + C::kBBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ProjBars<C::kStages>* bars = reinterpret_cast<ProjBars<C::kStages>*>(smem + C::kStages * kStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;       // head
  const int mt = blockIdx.y;      // tile of 128 tokens
  const int sp = blockIdx.z;      // slice of the head's output columns

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  const unsigned long long tmo = p.timeout_ns;
  int tma_issued = 0;
  bool mma_any = false;

  if (warp == 0) {
    if (lane == 0) {   // ------------------------------------------------ TMA producer
      for (int c = 0; c < C::kChunks; ++c) {
        const int s = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&bars->empty[s], ((c / C::kStages) - 1) & 1, tmo, abort_flag)) break;
        uint8_t* a = smem + s * kStage;
        uint8_t* b = a + C::kABytes;
        mbar_arrive_expect_tx(&bars->full[s], kStage);
        tma_load_3d(a, &tm_a, &bars->full[s], 64 * c, h, 128 * mt);   // token rows past n_tokens: zeros
        if constexpr (kAbsorb) {
#pragma unroll
          for (int j = 0; j < 2; ++j)   // W_UK[h] rows 64c..64c+63, output columns 128sp + 64j ..+63
            tma_load_3d(b + j * kBoxBytes, &tm_b, &bars->full[s], 128 * sp + 64 * j, 64 * c, h);
        } else {
          tma_load_3d(b, &tm_b, &bars->full[s], 64 * c, 32 * sp, h);  // W_UV[h] rows 32sp..+31, K chunk c
        }
        tma_issued = c + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {   // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = kAbsorb ? idesc_bf16_f32(128, 128, false, true) : idesc_bf16_f32(128, 32, false, false);
      bool all = true;
      for (int c = 0; c < C::kChunks; ++c) {
        const int s = c % C::kStages;
        if (!mbar_wait(&bars->full[s], (c / C::kStages) & 1, tmo, abort_flag)) {
          all = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kStage);
        const uint64_t dA = smem_desc_sw128(a, 16, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // K steps of 16 within the 64-wide chunk
          const uint32_t acc = (c > 0 || k > 0) ? 1u : 0u;
          if constexpr (kAbsorb) {
            // B MN-major: 64-column blocks 8 KB apart (LBO), K rows 128 B apart
            const uint64_t dB = smem_desc_sw128(a + C::kABytes, kBoxBytes, 1024);
            umma_bf16_ss(tmem, dA + static_cast<uint64_t>((k * 32) >> 4), dB + static_cast<uint64_t>((k * 2048) >> 4),
                         idesc, acc);
          } else {
            const uint64_t dB = smem_desc_sw128(a + C::kABytes, 16, 1024);
            umma_bf16_ss(tmem, dA + static_cast<uint64_t>((k * 32) >> 4), dB + static_cast<uint64_t>((k * 32) >> 4),
                         idesc, acc);
          }
        }
        mma_any = true;
        umma_commit(&bars->empty[s]);
      }
      if (all) umma_commit(&bars->done);
    }
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue (all four warps)
  if (mbar_wait(&bars->done, 0, tmo, abort_flag)) {
    tc_fence_after();
    const int row = warp * 32 + lane;
    const long long n = 128ll * mt + row;
    const bool valid = n < p.n_tokens;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    uint16_t* row_out = p.out + (n * p.heads + h) * static_cast<long long>(p.out_row);
    uint16_t* dst = row_out + C::kN * sp;
#pragma unroll 1
    for (int cc = 0; cc < C::kN / 32; ++cc) {
      float v[32];
      tmem_ld32(tmem + lane_base + 32u * cc, v);
      tc_wait_ld();
      if (valid) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __nv_bfloat162 b0 = __floats2bfloat162_rn(v[8 * q], v[8 * q + 1]);
          __nv_bfloat162 b1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
          __nv_bfloat162 b3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
          d4[q] = make_uint4(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1),
                             *reinterpret_cast<uint32_t*>(&b2), *reinterpret_cast<uint32_t*>(&b3));
        }
      }
    }
    if constexpr (kAbsorb) {   // the RoPE part passes through: q[n][h][128:192] -> q~[n][h][512:576]
      if (valid && sp == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(p.in + (n * p.heads + h) * 192ll + 128);
        uint4* d4 = reinterpret_cast<uint4*>(row_out + 512);
#pragma unroll
        for (int q = 0; q < 8; ++q) d4[q] = src[q];
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0 && p.flag != nullptr) atomicOr(p.flag, kFlagTimeout);
    if (warp == 0 && lane == 0) {   // let issued copies land before the memory goes away
      for (int c = 0; c < tma_issued; ++c) {
        volatile int never = 0;
        mbar_wait(&bars->full[c % C::kStages], (c / C::kStages) & 1, kProjDrainNs, &never);
      }
    }
    if (warp == 1 && lane == 0 && mma_any) {
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, kProjDrainNs, &never);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <bool kAbsorb>
cudaError_t proj_attrs() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(mla_proj_kernel<kAbsorb>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             proj_smem_bytes<kAbsorb>());
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_proj(bool absorb, const CUtensorMap& tm_a, const CUtensorMap& tm_b, const ProjParams& p,
                        cudaStream_t stream) {
  if (p.n_tokens == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(p.heads), static_cast<unsigned>((p.n_tokens + 127) / 128),
                  static_cast<unsigned>(absorb ? ProjCfg<true>::kSplits : ProjCfg<false>::kSplits));
  cudaError_t e;
  if (absorb) {
    if ((e = proj_attrs<true>()) != cudaSuccess) return e;
    mla_proj_kernel<true><<<grid, kProjThreads, proj_smem_bytes<true>(), stream>>>(tm_a, tm_b, p);
  } else {
    if ((e = proj_attrs<false>()) != cudaSuccess) return e;
    mla_proj_kernel<false><<<grid, kProjThreads, proj_smem_bytes<false>(), stream>>>(tm_a, tm_b, p);
  }
  return cudaGetLastError();
}

}  // namespace mla
