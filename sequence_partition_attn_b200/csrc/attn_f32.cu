// attn_f32.cu -- fp32 partition attention on the FMA units (true fp32 operands).
//
// Same per-partition state as the tensor-core path (DiTango web summary, Methodology 2,
// "State Composition"): for each selected (query tile, KV partition) pair,
// LSE_p(i) = ln sum_j exp(s_ij), O_p(i) = sum_j exp(s_ij - LSE_p(i)) v_j, s = scale*q.k.
// fp32 inputs need fp32 products: tf32 tensor-core inputs keep 10 mantissa bits, which
// misses a 1e-4 tolerance, so this path runs the dot products on the FMA pipe.
//
// Grid: x = 64-row query tile (over query groups with work), y = b*H + h, z = partition.
// A block holds 64 query rows; each row is owned by D/64 threads (64 dims each), which
// combine partial dot products with a shuffle.  Keys stream through shared memory in
// tiles of 32 with an online softmax (running max, running sum, rescaled accumulator).
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kRows = 64;
constexpr int kKeys = 32;

template <int D>
__global__ void __launch_bounds__(kRows * (D / 64)) attn_f32_kernel(const __grid_constant__ F32AttnParams prm) {
  constexpr int TPR = D / 64;
  __shared__ __align__(16) float sK[kKeys][D];
  __shared__ __align__(16) float sV[kKeys][D];
  const AttnTables& t = prm.t;
  const int bh = blockIdx.y;
  const int p = blockIdx.z;
  int qg = 0;
  while (qg + 1 < t.QG && t.tile_start[qg + 1] <= (int)blockIdx.x) ++qg;
  if (!fresh_bit(t.fresh_bits, qg, p)) return;

  const int row = threadIdx.x / TPR;
  const int half = threadIdx.x % TPR;
  const int q_row = t.qg_row0[qg] + (blockIdx.x - t.tile_start[qg]) * kRows + row;
  const bool row_ok = q_row < t.qg_row0[qg + 1];
  const int k0 = t.part_off[p], k1 = t.part_off[p + 1];
  const size_t head = static_cast<size_t>(bh) * prm.N;
  const size_t out_row = static_cast<size_t>(p) * prm.BH * prm.N + head + q_row;

  float q[64], o[64];
  const float* qp = prm.q + (head + (row_ok ? q_row : 0)) * D + half * 64;
#pragma unroll
  for (int d = 0; d < 64; d += 4) {
    const float4 v = *reinterpret_cast<const float4*>(qp + d);
    q[d] = v.x; q[d + 1] = v.y; q[d + 2] = v.z; q[d + 3] = v.w;
  }
#pragma unroll
  for (int d = 0; d < 64; ++d) o[d] = 0.0f;
  float m = -INFINITY, l = 0.0f;

  for (int key0 = k0; key0 < k1; key0 += kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeys * D / 4; idx += blockDim.x) {
      const int j = idx / (D / 4), c = (idx % (D / 4)) * 4;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (key0 + j < k1) {
        kv = *reinterpret_cast<const float4*>(prm.k + (head + key0 + j) * D + c);
        vv = *reinterpret_cast<const float4*>(prm.v + (head + key0 + j) * D + c);
      }
      *reinterpret_cast<float4*>(&sK[j][c]) = kv;
      *reinterpret_cast<float4*>(&sV[j][c]) = vv;
    }
    __syncthreads();
    float s[kKeys];
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float acc = 0.0f;
#pragma unroll
      for (int d = 0; d < 64; d += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(&sK[j][half * 64 + d]);
        acc = fmaf(q[d], kv.x, acc);
        acc = fmaf(q[d + 1], kv.y, acc);
        acc = fmaf(q[d + 2], kv.z, acc);
        acc = fmaf(q[d + 3], kv.w, acc);
      }
      if (TPR == 2) acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      s[j] = key0 + j < k1 ? acc * prm.scale : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    const float m_new = fmaxf(m, mt);
    const float alpha = expf(m - m_new);     // 0 on the first tile (m = -inf)
    l *= alpha;
#pragma unroll
    for (int d = 0; d < 64; ++d) o[d] *= alpha;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      const float pj = expf(s[j] - m_new);
      l += pj;
#pragma unroll
      for (int d = 0; d < 64; d += 4) {
        const float4 vv = *reinterpret_cast<const float4*>(&sV[j][half * 64 + d]);
        o[d] = fmaf(pj, vv.x, o[d]);
        o[d + 1] = fmaf(pj, vv.y, o[d + 1]);
        o[d + 2] = fmaf(pj, vv.z, o[d + 2]);
        o[d + 3] = fmaf(pj, vv.w, o[d + 3]);
      }
    }
    m = m_new;
  }

  if (!row_ok) return;
  float* dst = prm.o_part + out_row * D + half * 64;
  if (k1 <= k0) {                       // partition without keys
#pragma unroll
    for (int d = 0; d < 64; d += 4) *reinterpret_cast<float4*>(dst + d) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (half == 0) prm.lse_part[out_row] = -INFINITY;
    return;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int d = 0; d < 64; d += 4)
    *reinterpret_cast<float4*>(dst + d) = make_float4(o[d] * inv, o[d + 1] * inv, o[d + 2] * inv, o[d + 3] * inv);
  if (half == 0) prm.lse_part[out_row] = m + logf(l);
}

}  // namespace

int attn_f32_tile_rows() { return kRows; }

int launch_attn_f32(const F32AttnParams& prm, cudaStream_t st) {
  dim3 grid(prm.tiles_total, prm.BH, prm.t.P);
  if (prm.D == 64)
    attn_f32_kernel<64><<<grid, kRows, 0, st>>>(prm);
  else
    attn_f32_kernel<128><<<grid, kRows * 2, 0, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
