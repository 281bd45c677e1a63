// merge.cu -- LSE-weighted merge of attention states under a reuse mask, with fused
// partition importance, plus the stand-alone importance kernel and the reduction that
// turns per-block importance sums into means.
//
// Math (DiTango web summary, Methodology 2 "State Composition": output and log-sum-exp
// states compose associatively and commutatively; Methodology 1: fresh or reused per
// group, importance refreshed at anchor steps):
//   LSE(i) = ln sum_p exp(LSE_p(i)),   O(i) = sum_p exp(LSE_p(i) - LSE(i)) O_p(i),
//   w[qg][p] = mean over b, h, rows i of qg of exp(LSE_p(i) - LSE(i)),
// where the state of partition p is the fresh one when fresh[qg][p / G], else the cached.
//
// The merge is bound by HBM reads of the P states per row.  A block owns 128 rows of one
// query group of one (b, h):
//   phase 1  one thread per row reads the P log-sum-exps (coalesced across rows), forms
//            LSE with a running max, writes LSE and the P weights to shared memory;
//   phase 2  one warp per row streams the P state rows with 128-bit loads, 2..4 states
//            per warp iteration (a state row is D * elem bytes = 128..512 bytes), 8
//            iterations in flight, and reduces the partial sums with shuffles.
// Per-block importance sums go to a workspace [block][P]; reduce_w_kernel adds them per
// query group in a fixed order (deterministic) and divides by the row count.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kMR = 128;            // rows per block = threads per block
constexpr int kUnroll = 8;          // state loads in flight per lane

__device__ __forceinline__ int find_group(const int* start, int n, int x) {
  int g = 0;
  while (g + 1 < n && start[g + 1] <= x) ++g;
  return g;
}

template <typename T> struct Acc;
template <> struct Acc<float> {
  static constexpr int E = 4;
  __device__ static void add(float (&a)[8], const uint4& v, float w) {
    a[0] = fmaf(w, __uint_as_float(v.x), a[0]);
    a[1] = fmaf(w, __uint_as_float(v.y), a[1]);
    a[2] = fmaf(w, __uint_as_float(v.z), a[2]);
    a[3] = fmaf(w, __uint_as_float(v.w), a[3]);
  }
  __device__ static uint4 pack(const float (&a)[8]) {
    return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                      __float_as_uint(a[3]));
  }
};
template <> struct Acc<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static void add2(float& a0, float& a1, uint32_t u, float w) {
    a0 = fmaf(w, __uint_as_float(u << 16), a0);
    a1 = fmaf(w, __uint_as_float(u & 0xFFFF0000u), a1);
  }
  __device__ static void add(float (&a)[8], const uint4& v, float w) {
    add2(a[0], a[1], v.x, w);
    add2(a[2], a[3], v.y, w);
    add2(a[4], a[5], v.z, w);
    add2(a[6], a[7], v.w, w);
  }
  __device__ static uint4 pack(const float (&a)[8]) {
    return make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                      pack_bf16x2(a[6], a[7]));
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kMR) merge_kernel(const __grid_constant__ MergeParams prm) {
  extern __shared__ float sW[];                    // [P][kMR + 1] merged weights
  constexpr int kRowBytes = D * sizeof(T);
  constexpr int LPR = kRowBytes / 16;              // lanes per state row
  constexpr int SPW = 32 / LPR;                    // state rows per warp iteration
  const int P = prm.P;
  const int bh = blockIdx.x / prm.blocks_per_bh;
  const int blk = blockIdx.x - bh * prm.blocks_per_bh;
  const int qg = find_group(prm.blk_start, prm.QG, blk);
  const int r0 = prm.qg_row0[qg] + (blk - prm.blk_start[qg]) * kMR;
  const int nrows = min(kMR, prm.qg_row0[qg + 1] - r0);
  const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
  const size_t hrow0 = static_cast<size_t>(bh) * prm.N + r0;

  // Where each partition's state comes from for this block's query group: e >= 0, fresh
  // state e; e == -1, nothing (a partition of a reused group whose composed state sits in
  // the group's first slot); e <= -2, cached state -e - 2 (partition p, or KV group p/G
  // when the cache holds one composed state per group).
  __shared__ int s_state[PA_MAX_P];
  __shared__ int s_act[PA_MAX_P];                  // partitions with a state, in order
  __shared__ int s_nact;
  for (int p = threadIdx.x; p < P; p += kMR) {
    int e = p;
    if (!fresh_bit(prm.fresh_bits, qg, p))
      e = prm.cached_per_group ? (p % prm.G == 0 ? -(p / prm.G) - 2 : -1) : -p - 2;
    s_state[p] = e;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int p = 0; p < P; ++p)
      if (s_state[p] != -1) s_act[n++] = p;
    s_nact = n;
  }
  __syncthreads();
  const int nact = s_nact;

  // ---- phase 1: LSE and weights, one thread per row.  The log-sum-exps are loaded eight
  // at a time (independent loads in flight, not one latency per partition) and kept in
  // shared memory for the weights.
  {
    const int t = threadIdx.x;
    const bool ok = t < nrows;
    float m = -INFINITY, l = 0.0f;
    for (int p0 = 0; p0 < P; p0 += 8) {
      float Ls[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u;
        Ls[u] = -INFINITY;
        if (ok && p < P) {
          const int e = s_state[p];
          if (e != -1) {
            const float* src = e >= 0 ? prm.lse_fresh : prm.lse_cached;
            Ls[u] = src[(e >= 0 ? e : -e - 2) * BHN + hrow0 + t];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float L = Ls[u];
        if (L > m) {
          l = l * expf(m - L) + 1.0f;
          m = L;
        } else if (L > -INFINITY) {
          l += expf(L - m);
        }
        if (p0 + u < P) sW[(p0 + u) * (kMR + 1) + t] = L;
      }
    }
    const float lse = m > -INFINITY ? m + logf(l) : -INFINITY;
    if (ok) prm.lse[hrow0 + t] = lse;
    for (int p = 0; p < P; ++p) {
      const float L = sW[p * (kMR + 1) + t];
      sW[p * (kMR + 1) + t] = (ok && lse > -INFINITY && L > -INFINITY) ? expf(L - lse) : 0.0f;
    }
  }
  __syncthreads();
  if (prm.w_partial) {
    for (int p = threadIdx.x; p < P; p += kMR) {
      float s = 0.0f;
      for (int i = 0; i < nrows; ++i) s += sW[p * (kMR + 1) + i];
      prm.w_partial[static_cast<size_t>(blockIdx.x) * P + p] = s;
    }
  }

  // ---- phase 2: weighted sum of the state rows
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPR, slot = lane / LPR;
  const uint8_t* of = static_cast<const uint8_t*>(prm.o_fresh);
  const uint8_t* oc = static_cast<const uint8_t*>(prm.o_cached);
  if (SPW > 1 && nact <= kUnroll) {
    // Few states per row: each group of LPR lanes takes a row of its own and loads all of
    // its states at once, so a warp keeps SPW rows' loads in flight (no reduction across
    // lane groups is needed: lane `sub` owns chunk `sub` of its row).
    for (int i = warp * SPW + slot; i < nrows; i += (kMR / 32) * SPW) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const size_t rowoff = (hrow0 + i) * kRowBytes + sub * 16;
      uint4 v[kUnroll];
      float wt[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        wt[u] = 0.0f;
        v[u] = make_uint4(0, 0, 0, 0);
        if (u < nact) {
          const int p = s_act[u];
          const int e = s_state[p];
          wt[u] = sW[p * (kMR + 1) + i];
          const uint8_t* base = e >= 0 ? of : oc;
          v[u] = __ldg(reinterpret_cast<const uint4*>(base + (e >= 0 ? e : -e - 2) * BHN * kRowBytes + rowoff));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) Acc<T>::add(acc, v[u], wt[u]);
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(prm.o) + rowoff) = Acc<T>::pack(acc);
    }
    return;
  }
  // One warp per row.
  for (int i = warp; i < nrows; i += kMR / 32) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const size_t rowoff = (hrow0 + i) * kRowBytes + sub * 16;
    // Only the partitions that contribute a state are visited (a composed cache leaves
    // most slots of a reused group empty), so every load slot in flight is a real one.
    for (int k0 = 0; k0 < nact; k0 += SPW * kUnroll) {
      uint4 v[kUnroll];
      float wt[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * SPW + slot;
        wt[u] = 0.0f;
        v[u] = make_uint4(0, 0, 0, 0);
        if (k < nact) {
          const int p = s_act[k];
          const int e = s_state[p];
          wt[u] = sW[p * (kMR + 1) + i];
          const uint8_t* base = e >= 0 ? of : oc;
          v[u] = __ldg(reinterpret_cast<const uint4*>(base + (e >= 0 ? e : -e - 2) * BHN * kRowBytes + rowoff));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) Acc<T>::add(acc, v[u], wt[u]);
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < Acc<T>::E; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (slot == 0)
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(prm.o) + rowoff) = Acc<T>::pack(acc);
  }
}

__global__ void __launch_bounds__(kMR) importance_kernel(const __grid_constant__ ImportanceParams prm) {
  __shared__ float sPart[kMR / 32][PA_MAX_P];
  const int P = prm.P;
  const int bh = blockIdx.x / prm.blocks_per_bh;
  const int blk = blockIdx.x - bh * prm.blocks_per_bh;
  const int qg = find_group(prm.blk_start, prm.QG, blk);
  const int r0 = prm.qg_row0[qg] + (blk - prm.blk_start[qg]) * kMR;
  const int nrows = min(kMR, prm.qg_row0[qg + 1] - r0);
  const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
  const size_t hrow = static_cast<size_t>(bh) * prm.N + r0 + threadIdx.x;
  const bool ok = static_cast<int>(threadIdx.x) < nrows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float L = ok ? prm.lse[hrow] : -INFINITY;
  for (int p = 0; p < P; ++p) {
    float w = (ok && L > -INFINITY) ? expf(prm.lse_part[p * BHN + hrow] - L) : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if (lane == 0) sPart[warp][p] = w;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += kMR) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kMR / 32; ++w) s += sPart[w][p];
    prm.w_partial[static_cast<size_t>(blockIdx.x) * P + p] = s;
  }
}

// One block per (query group, partition): the threads stride over the group's (b*h,
// row block) partial sums in a fixed assignment and add them in fp64, then a fixed-shape
// tree adds the threads' sums -- the same order on every run (deterministic).
constexpr int kRT = 256;

__global__ void __launch_bounds__(kRT) reduce_w_kernel(const __grid_constant__ ReduceWParams prm) {
  __shared__ double s_sum[kRT];
  const int qg = blockIdx.x / prm.P, p = blockIdx.x - qg * prm.P;
  const int b0 = prm.blk_start[qg], nb = prm.blk_start[qg + 1] - b0;
  const long long E = static_cast<long long>(prm.BH) * nb;
  double acc = 0.0;
  for (long long e = threadIdx.x; e < E; e += kRT) {
    const long long bh = e / nb;
    const long long b = e - bh * nb;
    acc += prm.w_partial[(bh * prm.blocks_per_bh + b0 + b) * prm.P + p];
  }
  s_sum[threadIdx.x] = acc;
  __syncthreads();
  for (int off = kRT / 2; off > 0; off >>= 1) {
    if (static_cast<int>(threadIdx.x) < off) s_sum[threadIdx.x] += s_sum[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) prm.w[qg * prm.P + p] = static_cast<float>(s_sum[0] * prm.inv_count[qg]);
}

// Compose: the states of every `factor` consecutive partitions merged into one (DiTango
// web summary, Methodology 2, "Dynamic Group Compose": coarser cached states without
// recomputation).  One block per (output group c, b*h, kCR rows): phase 1 forms each
// row's LSE over the group's partitions and the weights exp(LSE_p - LSE); phase 2 gives
// every thread 16-byte chunks of kItems (row, chunk) items and, partition by partition,
// keeps kItems loads in flight.
constexpr int kCThreads = 256;
constexpr int kCR = 128;            // rows per compose block

template <typename T, int D>
__global__ void __launch_bounds__(kCThreads) compose_kernel(const __grid_constant__ ComposeParams prm) {
  extern __shared__ float sW[];                    // [factor][kCR + 1]
  constexpr int kCh = D * static_cast<int>(sizeof(T)) / 16;   // chunks per state row
  constexpr int kItems = kCR * kCh / kCThreads;
  const int per_c = prm.BH * prm.nblk;
  const int c = blockIdx.x / per_c;
  const int rem = blockIdx.x - c * per_c;
  const int bh = rem / prm.nblk;
  const int r0 = (rem - bh * prm.nblk) * kCR;
  const int nrows = min(kCR, prm.N - r0);
  const int p0 = c * prm.factor;
  const int np = min(prm.factor, prm.P - p0);
  const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
  const size_t hrow0 = static_cast<size_t>(bh) * prm.N + r0;

  if (threadIdx.x < kCR) {
    const int t = threadIdx.x;
    const bool ok = t < nrows;
    float m = -INFINITY, l = 0.0f;
    if (ok) {
      for (int g = 0; g < np; ++g) {
        const float L = prm.lse_part[(p0 + g) * BHN + hrow0 + t];
        if (L > m) {
          l = l * expf(m - L) + 1.0f;
          m = L;
        } else if (L > -INFINITY) {
          l += expf(L - m);
        }
      }
    }
    const float lse = m > -INFINITY ? m + logf(l) : -INFINITY;
    if (ok) prm.lse_group[c * BHN + hrow0 + t] = lse;
    for (int g = 0; g < np; ++g) {
      float w = 0.0f;
      if (ok && lse > -INFINITY) w = expf(prm.lse_part[(p0 + g) * BHN + hrow0 + t] - lse);
      sW[g * (kCR + 1) + t] = w;
    }
  }
  __syncthreads();

  const uint4* src = static_cast<const uint4*>(prm.o_part);
  uint4* dst = static_cast<uint4*>(prm.o_group);
  const int nitems = nrows * kCh;
  float acc[kItems][8];
#pragma unroll
  for (int k = 0; k < kItems; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.0f;
  const bool full = nitems == kCR * kCh;            // every item valid: unguarded loads
  for (int g = 0; g < np; ++g) {
    const size_t base = ((p0 + g) * BHN + hrow0) * kCh;
    uint4 v[kItems];
    if (full) {
#pragma unroll
      for (int k = 0; k < kItems; ++k) v[k] = __ldg(src + base + threadIdx.x + k * kCThreads);
    } else {
#pragma unroll
      for (int k = 0; k < kItems; ++k) {
        const int idx = threadIdx.x + k * kCThreads;
        v[k] = idx < nitems ? __ldg(src + base + idx) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int idx = threadIdx.x + k * kCThreads;
      const float w = idx < nitems ? sW[g * (kCR + 1) + idx / kCh] : 0.0f;
      Acc<T>::add(acc[k], v[k], w);
    }
  }
  const size_t obase = (c * BHN + hrow0) * kCh;
#pragma unroll
  for (int k = 0; k < kItems; ++k) {
    const int idx = threadIdx.x + k * kCThreads;
    if (idx < nitems) dst[obase + idx] = Acc<T>::pack(acc[k]);
  }
}

template <typename T, int D>
int compose_impl(const ComposeParams& prm, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(prm.factor) * (kCR + 1) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(compose_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  const long long C = (prm.P + prm.factor - 1) / prm.factor;
  const long long blocks = C * prm.BH * prm.nblk;
  compose_kernel<T, D><<<static_cast<unsigned>(blocks), kCThreads, smem, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

template <typename T, int D>
int merge_impl(const MergeParams& prm, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(prm.P) * (kMR + 1) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(merge_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  const long long blocks = static_cast<long long>(prm.BH) * prm.blocks_per_bh;
  merge_kernel<T, D><<<static_cast<unsigned>(blocks), kMR, smem, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int merge_rows_per_block() { return kMR; }
int compose_rows_per_block() { return kCR; }

int launch_merge(const MergeParams& prm, int dtype, cudaStream_t st) {
  if (dtype == PA_BF16) return prm.D == 64 ? merge_impl<__nv_bfloat16, 64>(prm, st) : merge_impl<__nv_bfloat16, 128>(prm, st);
  return prm.D == 64 ? merge_impl<float, 64>(prm, st) : merge_impl<float, 128>(prm, st);
}

int launch_compose(const ComposeParams& prm, int dtype, int D, cudaStream_t st) {
  if (dtype == PA_BF16) return D == 64 ? compose_impl<__nv_bfloat16, 64>(prm, st) : compose_impl<__nv_bfloat16, 128>(prm, st);
  return D == 64 ? compose_impl<float, 64>(prm, st) : compose_impl<float, 128>(prm, st);
}

int launch_importance(const ImportanceParams& prm, cudaStream_t st) {
  const long long blocks = static_cast<long long>(prm.BH) * prm.blocks_per_bh;
  importance_kernel<<<static_cast<unsigned>(blocks), kMR, 0, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

int launch_reduce_w(const ReduceWParams& prm, cudaStream_t st) {
  reduce_w_kernel<<<prm.QG * prm.P, kRT, 0, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
