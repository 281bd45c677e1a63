// relayout.cu -- sequence-major -> head-major permutation, the single-device stand-in for
// the Ulysses all-to-all (SwiftFusion web summary, Methodology 2 "Torus Attention": the
// all-to-all is cut into sequence chunks so that compute on moved chunks overlaps the
// movement of later ones).
//
// dst[h][n][:] = src[n][h][:] for n in [n0, n1).  A token-head row (D * elem bytes) moves
// whole, as 16-byte pieces: reads walk the source linearly (coalesced), writes land in
// full contiguous rows of the destination.  Pure HBM traffic: 2 * rows * row bytes.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) relayout_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                            long long n0, long long total, int N, int H,
                                                            int ppr) {
  const long long stride = static_cast<long long>(gridDim.x) * kThreads;
  const long long src0 = n0 * H * ppr;
  for (long long base = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long idx = base + u * stride;
      if (idx < total) v[u] = __ldg(src + src0 + idx);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long idx = base + u * stride;
      if (idx < total) {
        const long long rowi = idx / ppr;
        const int piece = static_cast<int>(idx - rowi * ppr);
        const long long n = n0 + rowi / H;
        const int h = static_cast<int>(rowi % H);
        dst[(static_cast<long long>(h) * N + n) * ppr + piece] = v[u];
      }
    }
  }
}

}  // namespace

int launch_relayout(const void* src, void* dst, long long n0, long long n1, int N, int H, int row_bytes,
                    int sm_count, cudaStream_t st) {
  const int ppr = row_bytes / 16;
  const long long total = (n1 - n0) * H * ppr;
  if (total <= 0) return 0;
  long long blocks = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const long long cap = static_cast<long long>(sm_count) * 8;
  if (blocks > cap) blocks = cap;
  relayout_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), n0, total, N, H, ppr);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
