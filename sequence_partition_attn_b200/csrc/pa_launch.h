// pa_launch.h -- host-side launchers of libpa's kernels (internal; the public ABI is pa.h).
// Each returns a cudaError_t value (0 on success).
#pragma once

#include <cuda_runtime.h>

#include "pa_device.cuh"

namespace pa {

// One CTA per work unit: CTA i takes unit i, or unit ord->unit[i] when `ord` is given.
int launch_attn_tc(const TcParams& prm, const TcUnitOrder* ord, int units, cudaStream_t st);
int attn_tc_tile_rows();

int launch_attn_f32(const F32AttnParams& prm, cudaStream_t st);
int attn_f32_tile_rows();

int launch_merge(const MergeParams& prm, int dtype, cudaStream_t st);
int merge_rows_per_block();
int launch_importance(const ImportanceParams& prm, cudaStream_t st);
int launch_reduce_w(const ReduceWParams& prm, cudaStream_t st);

int compose_rows_per_block();
int launch_compose(const ComposeParams& prm, int dtype, int D, cudaStream_t st);

int launch_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t st);

int drift_rows_per_block();
int launch_drift(const DriftParams& prm, int dtype, int D, cudaStream_t st);
int launch_reduce_pair(const ReducePairParams& prm, cudaStream_t st);

// dst[h][dst_n0 + n - n0][:] = src[n][h][:], n in [n0, n1); dst has dst_N tokens per head.
int launch_relayout(const void* src, void* dst, long long n0, long long n1, long long dst_n0, int dst_N,
                    int H, int row_bytes, int sm_count, cudaStream_t st);

}  // namespace pa
