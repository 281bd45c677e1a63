// drift.cu -- state drift between two sets of attention states, the measurement behind
// online error prediction between anchor steps (DiTango web summary, Methodology 1,
// "Online Prediction": the change of the local states, which are always computed, stands
// in for the drift of the reused remote states).
//
// For every selected pair (query group qg, partition p):
//   d2[qg][p] = sum over batch, heads, rows of qg, channels of (O_new - O_ref)^2,
//   r2[qg][p] = the same sum of O_ref^2.
// Bound by HBM reads of the two state sets.  A block owns up to 128 rows of one query group
// of one (b, h); the rows of a partition's states are contiguous, so the block reads
// nrows * D * elem bytes per selected partition with 16-byte coalesced loads, 8 per
// tensor in flight per thread.  Warps keep per-partition sums in shared memory and the
// block adds them once at the end; per-block sums go to a workspace and are added per
// query group in a fixed order (deterministic).
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kRows = 128;
constexpr int kThreads = 256;
constexpr int kBatch = 8;

template <typename T> struct Elems;
template <> struct Elems<float> {
  __device__ static void acc(const uint4& a, const uint4& b, float& dd, float& rr) {
    const float av[4] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w)};
    const float bv[4] = {__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float d = av[i] - bv[i];
      dd = fmaf(d, d, dd);
      rr = fmaf(bv[i], bv[i], rr);
    }
  }
};
template <> struct Elems<__nv_bfloat16> {
  __device__ static void acc(const uint4& a, const uint4& b, float& dd, float& rr) {
    const uint32_t au[4] = {a.x, a.y, a.z, a.w}, bu[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a0 = __uint_as_float(au[i] << 16), a1 = __uint_as_float(au[i] & 0xFFFF0000u);
      const float b0 = __uint_as_float(bu[i] << 16), b1 = __uint_as_float(bu[i] & 0xFFFF0000u);
      dd = fmaf(a0 - b0, a0 - b0, dd);
      dd = fmaf(a1 - b1, a1 - b1, dd);
      rr = fmaf(b0, b0, rr);
      rr = fmaf(b1, b1, rr);
    }
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) drift_kernel(const __grid_constant__ DriftParams prm) {
  constexpr int kChunks = D * sizeof(T) / 16;      // 16-byte pieces per state row
  constexpr int kWarps = kThreads / 32;
  // Per-warp sums of every partition; the block adds them once at the end, so warps run
  // ahead from one partition to the next without a block barrier in between.
  __shared__ float s_red[2][PA_MAX_P][kWarps];
  const int bh = blockIdx.x / prm.blocks_per_bh;
  const int blk = blockIdx.x - bh * prm.blocks_per_bh;
  int qg = 0;
  while (qg + 1 < prm.QG && prm.blk_start[qg + 1] <= blk) ++qg;
  const int r0 = prm.qg_row0[qg] + (blk - prm.blk_start[qg]) * kRows;
  const int nrows = min(kRows, prm.qg_row0[qg + 1] - r0);
  const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
  const size_t first = static_cast<size_t>(bh) * prm.N + r0;     // first row of the block
  const uint4* a = static_cast<const uint4*>(prm.o_new);
  const uint4* b = static_cast<const uint4*>(prm.o_ref);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = nrows * kChunks;
  for (int p = 0; p < prm.P; ++p) {
    float dd = 0.0f, rr = 0.0f;
    if (fresh_bit(prm.sel_bits, qg, p / prm.G)) {
      const size_t base = (static_cast<size_t>(p) * BHN + first) * kChunks;
      // kBatch chunks of each tensor in flight per thread.
      for (int i0 = 0; i0 < n; i0 += kBatch * kThreads) {
        uint4 va[kBatch], vb[kBatch];
        if (i0 + kBatch * kThreads <= n) {          // whole batch in range: unguarded loads
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            va[k] = __ldg(a + base + i0 + threadIdx.x + k * kThreads);
            vb[k] = __ldg(b + base + i0 + threadIdx.x + k * kThreads);
          }
        } else {
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int idx = i0 + threadIdx.x + k * kThreads;
            va[k] = idx < n ? __ldg(a + base + idx) : make_uint4(0, 0, 0, 0);
            vb[k] = idx < n ? __ldg(b + base + idx) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) Elems<T>::acc(va[k], vb[k], dd, rr);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        dd += __shfl_xor_sync(0xffffffffu, dd, off);
        rr += __shfl_xor_sync(0xffffffffu, rr, off);
      }
    }
    if (lane == 0) {
      s_red[0][p][warp] = dd;
      s_red[1][p][warp] = rr;
    }
  }
  __syncthreads();
  float* out = prm.partial + static_cast<size_t>(blockIdx.x) * 2 * prm.P;
  for (int p = threadIdx.x; p < prm.P; p += kThreads) {
    float sd = 0.0f, sr = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      sd += s_red[0][p][w];
      sr += s_red[1][p][w];
    }
    out[p] = sd;
    out[prm.P + p] = sr;
  }
}

// One block per (query group, partition): fixed assignment of the (b*h, row block)
// partial sums to threads, fp64 sums, fixed-shape tree (deterministic).
constexpr int kRT = 256;

__global__ void __launch_bounds__(kRT) reduce_pair_kernel(const __grid_constant__ ReducePairParams prm) {
  __shared__ double s_sum[2][kRT];
  const int qg = blockIdx.x / prm.P, p = blockIdx.x - qg * prm.P;
  const int b0 = prm.blk_start[qg], nb = prm.blk_start[qg + 1] - b0;
  const long long E = static_cast<long long>(prm.BH) * nb;
  double sd = 0.0, sr = 0.0;
  for (long long e = threadIdx.x; e < E; e += kRT) {
    const long long bh = e / nb;
    const long long b = e - bh * nb;
    const float* part = prm.partial + (bh * prm.blocks_per_bh + b0 + b) * 2 * prm.P;
    sd += part[p];
    sr += part[prm.P + p];
  }
  s_sum[0][threadIdx.x] = sd;
  s_sum[1][threadIdx.x] = sr;
  __syncthreads();
  for (int off = kRT / 2; off > 0; off >>= 1) {
    if (static_cast<int>(threadIdx.x) < off) {
      s_sum[0][threadIdx.x] += s_sum[0][threadIdx.x + off];
      s_sum[1][threadIdx.x] += s_sum[1][threadIdx.x + off];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    prm.d2[qg * prm.P + p] = static_cast<float>(s_sum[0][0]);
    prm.r2[qg * prm.P + p] = static_cast<float>(s_sum[1][0]);
  }
}

template <typename T, int D>
int drift_impl(const DriftParams& prm, cudaStream_t st) {
  const long long blocks = static_cast<long long>(prm.BH) * prm.blocks_per_bh;
  drift_kernel<T, D><<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int drift_rows_per_block() { return kRows; }

int launch_drift(const DriftParams& prm, int dtype, int D, cudaStream_t st) {
  if (dtype == PA_BF16) return D == 64 ? drift_impl<__nv_bfloat16, 64>(prm, st) : drift_impl<__nv_bfloat16, 128>(prm, st);
  return D == 64 ? drift_impl<float, 64>(prm, st) : drift_impl<float, 128>(prm, st);
}

int launch_reduce_pair(const ReducePairParams& prm, cudaStream_t st) {
  reduce_pair_kernel<<<prm.QG * prm.P, kRT, 0, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
