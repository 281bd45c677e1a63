// relayout.cu -- sequence-major -> head-major permutation, the single-device stand-in for
// the Ulysses all-to-all (SwiftFusion web summary, Methodology 2 "Torus Attention": the
// all-to-all is cut into sequence chunks so that compute on moved chunks overlaps the
// movement of later ones).
//
// dst[h][dst_n0 + n - n0][:] = src[n][h][:] for n in [n0, n1), dst holding dst_N tokens
// per head (the whole-sequence relayout has dst_n0 = n0 and dst_N = N; a piece of a
// sequence-parallel all-to-all lands at its own token offset of a longer head-major
// tensor).  A token-head row (D * elem bytes) moves whole, as 16-byte pieces: reads walk
// the source linearly (coalesced), writes land in full contiguous rows of the
// destination.  Pure HBM traffic: 2 * rows * row bytes.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// Thread t of the grid copies piece (t mod ppr) of rows r, r + dr, r + 2 dr, ... where
// r = t / ppr and dr = grid threads / ppr (the block size is a multiple of ppr, so every
// thread keeps its piece).  Row r = n' * H + h is token n0 + n', head h; (n', h) of each of the
// kUnroll rows in flight advance by a constant step with one carry, so the loop does no
// division.
__global__ void __launch_bounds__(1024) relayout_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                        long long n0, long long dst_n0, long long rows, int N,
                                                        int H, int ppr) {
  const long long gthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int piece = static_cast<int>(t % ppr);
  const long long dr = gthreads / ppr;                 // rows per grid step
  const long long step = dr * kUnroll;                 // rows per loop iteration
  const long long step_n = step / H;
  const int step_h = static_cast<int>(step % H);
  long long r[kUnroll], n[kUnroll];
  int h[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    r[u] = t / ppr + u * dr;
    n[u] = r[u] / H;
    h[u] = static_cast<int>(r[u] - n[u] * H);
  }
  const uint4* s0 = src + n0 * H * ppr + piece;
  uint4* d0 = dst + dst_n0 * ppr + piece;
  while (r[0] < rows) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (r[u] < rows) v[u] = __ldg(s0 + r[u] * ppr);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (r[u] < rows) d0[(static_cast<long long>(h[u]) * N + n[u]) * ppr] = v[u];
      r[u] += step;
      n[u] += step_n;
      h[u] += step_h;
      if (h[u] >= H) {
        h[u] -= H;
        ++n[u];
      }
    }
  }
}

}  // namespace

int launch_relayout(const void* src, void* dst, long long n0, long long n1, long long dst_n0, int dst_N,
                    int H, int row_bytes, int sm_count, cudaStream_t st) {
  const int ppr = row_bytes / 16;                    // 16-byte pieces per row
  if (ppr < 1 || ppr > 1024) return static_cast<int>(cudaErrorInvalidValue);
  const int threads = ppr >= kThreads ? ppr : (kThreads / ppr) * ppr;   // a multiple of ppr
  const long long rows = (n1 - n0) * H;
  if (rows <= 0) return 0;
  long long blocks = (rows * ppr + static_cast<long long>(threads) * kUnroll - 1) / (static_cast<long long>(threads) * kUnroll);
  // up to 32 blocks per SM (8 resident at once): the grid-stride loop then ends more evenly
  // (228 / 233 / 242 us on [115200][24][128] bf16 with 32 / 16 / 8 per SM)
  const long long cap = static_cast<long long>(sm_count) * 32;
  if (blocks > cap) blocks = cap;
  relayout_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), n0, dst_n0, rows, dst_N, H, ppr);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
