// Host-side launchers of the decode kernels (internal to libmla_decode.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_common.cuh"

namespace mla {

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream);

// Grid: row_tiles * c_max clusters of 2 CTAs; p.tile_rows (64 or 128) and
// p.fp8 pick the variant. tm_q: query rope box; tm_kv: bf16 page boxes (or fp8
// latent boxes); tm_kv2: fp8 rope boxes (unused for bf16).
cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_kv2,
                          const DecodeParams& p, cudaStream_t stream);
// Co-resident 2-CTA clusters of one variant (also raises that variant's dynamic
// shared-memory limit on the current device).
cudaError_t decode_max_active_clusters(int tile_rows, bool fp8, int* clusters);

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

cudaError_t launch_cascade_prep(const CascadeParams& p, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);

// absorb: tm_a = q nope boxes, tm_b = W_UK boxes; project: tm_a = o boxes, tm_b = W_UV boxes.
cudaError_t launch_proj(bool absorb, const CUtensorMap& tm_a, const CUtensorMap& tm_b, const ProjParams& p,
                        cudaStream_t stream);

// Records `status` and a printf-style message as this thread's last error
// (read back by mla_get_last_error); returns `status`.
int set_last_error(int status, const char* fmt, ...);

}  // namespace mla
