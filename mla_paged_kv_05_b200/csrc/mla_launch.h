// Host-side launchers of the decode kernels (internal to libmla_decode.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_common.cuh"

namespace mla {

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream);

// Grid: row_tiles * c_max clusters of 2 CTAs; p.tile_rows (64 or 128) picks the variant.
cudaError_t launch_decode_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const DecodeParams& p,
                               cudaStream_t stream);
// Co-resident 2-CTA clusters of the variant with `tile_rows` query rows per tile
// (also raises that variant's dynamic shared-memory limit on the current device).
cudaError_t decode_bf16_max_active_clusters(int tile_rows, int* clusters);

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

// Records `status` and a printf-style message as this thread's last error
// (read back by mla_get_last_error); returns `status`.
int set_last_error(int status, const char* fmt, ...);

}  // namespace mla
