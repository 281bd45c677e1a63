// attn_tc.cu -- bf16 partition attention on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every (query tile, KV partition) pair selected as fresh, the attention
// state of the partition: LSE_p(i) = ln sum_j exp(s_ij) and
// O_p(i) = sum_j exp(s_ij - LSE_p(i)) v_j over the partition's valid keys, s = scale*q.k.
// This is the per-partition state of the DiTango web summary (Methodology 2, "State
// Composition"; the ring-based group state computation iterates partitions the same way).
//
// One CTA owns one 128-row query tile of one (batch, head) and walks every fresh KV
// partition of its query group in order.  The running softmax restarts at each partition
// boundary, where the epilogue writes (O_p, LSE_p).
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then K and V tiles of 128 keys into a 2-stage ring.
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into TMEM, then O += P V into TMEM.
//   warps 2..5  softmax warpgroup, one query row per thread (TMEM lane = row): reads S
//               from TMEM, masks keys past the partition end, keeps the running max and
//               sum in the log2 domain, rescales O in TMEM when the max grows, writes
//               P (bf16) to shared memory for the PV product, and runs the epilogue.
//
// Overlap: the MMA warp issues S(j+1) as soon as the softmax has released S(j), so the
// exponentials of tile j+1 run while PV(j) occupies the tensor pipe.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kBM = 128;        // query rows per tile (MMA M)
constexpr int kBN = 128;        // keys per tile (MMA N of S, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 192;
constexpr int kAtomBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16): one swizzle-128B box

template <int D>
struct Layout {
  static constexpr int kAtoms = D / 64;
  static constexpr int kTileBytes = kAtoms * kAtomBytes;   // a 128 x D bf16 tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kP = kV + kStages * kTileBytes;
  static constexpr int kBar = kP + 2 * kAtomBytes;         // P: 128 rows x 128 keys bf16
  enum { Q_FULL = 0, K_FULL = 1, V_FULL = K_FULL + kStages, KV_EMPTY = V_FULL + kStages,
         S_FULL = KV_EMPTY + kStages, P_FULL, O_DONE, NBAR };
  static constexpr int kTmemSlot = kBar + NBAR * 8;
  static constexpr int kAbort = kTmemSlot + 8;
  static constexpr int kUsed = kAbort + 8;
  static constexpr int kSmemBytes = kUsed + 1024;          // slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 256;               // S: 128 columns, O: D columns
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(128 + D <= (int)kTmemCols, "TMEM budget");
};

constexpr float kLn2 = 0.6931471805599453f;

// Next partition >= from that is fresh for query group qg and holds at least one key.
__device__ __forceinline__ int next_part(const AttnTables& t, int qg, int from) {
  for (int p = from; p < t.P; ++p)
    if (fresh_bit(t.fresh_bits, qg, p) && t.part_off[p + 1] > t.part_off[p]) return p;
  return t.P;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams prm) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kAbort);
  int* status = prm.status;
  const AttnTables& t = prm.t;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Decode the work unit: (b*H + h, query group, 128-row tile of the group).
  const int bh = blockIdx.x / prm.tiles_total;
  const int tix = blockIdx.x - bh * prm.tiles_total;
  int qg = 0;
  while (qg + 1 < t.QG && t.tile_start[qg + 1] <= tix) ++qg;
  const int q_row0 = t.qg_row0[qg] + (tix - t.tile_start[qg]) * kBM;
  const int q_end = t.qg_row0[qg + 1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NBAR; ++i) mbar_init(bar(i), i == L::P_FULL ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kTmemSlot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);
  const uint32_t tS = tmem;          // columns [0, 128)
  const uint32_t tO = tmem + 128;    // columns [128, 128 + D)

  const uint32_t sQ = base + L::kQ;
  const uint32_t sP = base + L::kP;
  auto sK = [&](int s) { return base + L::kK + (uint32_t)s * L::kTileBytes; };
  auto sV = [&](int s) { return base + L::kV + (uint32_t)s * L::kTileBytes; };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch(&prm.tm_q);
      tma_prefetch(&prm.tm_k);
      tma_prefetch(&prm.tm_v);
      mbar_expect_tx(bar(L::Q_FULL), L::kTileBytes);
      for (int a = 0; a < L::kAtoms; ++a)
        tma_load_3d(sQ + a * kAtomBytes, &prm.tm_q, a * 64, q_row0, bh, bar(L::Q_FULL));
      int j = 0;
      bool ok = true;
      for (int p = next_part(t, qg, 0); ok && p < t.P; p = next_part(t, qg, p + 1)) {
        const int k1 = t.part_off[p + 1];
        for (int key = t.part_off[p]; key < k1; key += kBN, ++j) {
          const int s = j % kStages;
          if (j >= kStages &&
              !mbar_wait(bar(L::KV_EMPTY + s), ((j / kStages) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(L::K_FULL + s), L::kTileBytes);
          for (int a = 0; a < L::kAtoms; ++a)
            tma_load_3d(sK(s) + a * kAtomBytes, &prm.tm_k, a * 64, key, bh, bar(L::K_FULL + s));
          mbar_expect_tx(bar(L::V_FULL + s), L::kTileBytes);
          for (int a = 0; a < L::kAtoms; ++a)
            tma_load_3d(sV(s) + a * kAtomBytes, &prm.tm_v, a * 64, key, bh, bar(L::V_FULL + s));
        }
      }
      // Every load issued must have landed before the CTA may exit.
      mbar_drain(bar(L::Q_FULL), 0);
      for (int jj = (j > kStages ? j - kStages : 0); jj < j; ++jj) {
        mbar_drain(bar(L::K_FULL + jj % kStages), (jj / kStages) & 1);
        mbar_drain(bar(L::V_FULL + jj % kStages), (jj / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(kBM, kBN, false, false);   // Q K-major, K K-major
      constexpr uint32_t kIdPV = idesc_bf16(kBM, D, false, true);     // P K-major, V MN-major
      int T = 0;
      for (int p = next_part(t, qg, 0); p < t.P; p = next_part(t, qg, p + 1))
        T += (t.part_off[p + 1] - t.part_off[p] + kBN - 1) / kBN;
      auto issue_s = [&](int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
          mma_bf16_ss(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK(s) + off, 16, 1024),
                      kIdS, kk > 0);
        }
      };
      bool ok = mbar_wait(bar(L::Q_FULL), 0, abort_flag, status);
      int j = 0;
      if (ok && T > 0) {
        ok = mbar_wait(bar(L::K_FULL + 0), 0, abort_flag, status);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          mma_commit(bar(L::S_FULL));
        }
        int p = next_part(t, qg, 0);
        int key = t.part_off[p];
        for (; ok && j < T; ++j) {
          const bool first = key == t.part_off[p];
          if (!mbar_wait(bar(L::P_FULL), j & 1, abort_flag, status)) { ok = false; break; }
          tc_fence_after();
          if (j + 1 < T) {
            const int s1 = (j + 1) % kStages;
            if (!mbar_wait(bar(L::K_FULL + s1), ((j + 1) / kStages) & 1, abort_flag, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(s1);
            mma_commit(bar(L::S_FULL));
          }
          const int s = j % kStages;
          if (!mbar_wait(bar(L::V_FULL + s), (j / kStages) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            mma_bf16_ss(tO, smem_desc_sw128(sP + aoff, 16, 1024),
                        smem_desc_sw128(sV(s) + kk * 16 * 128, kAtomBytes, 1024), kIdPV,
                        (first && kk == 0) ? 0u : 1u);
          }
          mma_commit(bar(L::O_DONE));
          mma_commit(bar(L::KV_EMPTY + s));
          key += kBN;
          if (key >= t.part_off[p + 1]) {
            p = next_part(t, qg, p + 1);
            key = p < t.P ? t.part_off[p] : 0;
          }
        }
      }
      // The last commits must have arrived before the CTA may exit.
      for (int jj = (j > kStages ? j - kStages : 0); jj < j; ++jj)
        mbar_drain(bar(L::KV_EMPTY + jj % kStages), (jj / kStages) & 1);
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroup
    const int wq = warp & 3;                       // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;
    const int q_row = q_row0 + row;
    const bool row_ok = q_row < q_end;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
    __nv_bfloat16* o_part = static_cast<__nv_bfloat16*>(prm.o_part);

    // Fresh partitions without keys: LSE = -inf, O = 0.
    for (int p = 0; p < t.P; ++p) {
      if (!fresh_bit(t.fresh_bits, qg, p) || t.part_off[p + 1] > t.part_off[p] || !row_ok) continue;
      const size_t r = static_cast<size_t>(p) * BHN + static_cast<size_t>(bh) * prm.N + q_row;
      uint4* dst = reinterpret_cast<uint4*>(o_part + r * D);
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      prm.lse_part[r] = -INFINITY;
    }

    auto epilogue = [&](int p, float m, float l) {
      const float inv = 1.0f / l;
      const size_t r = static_cast<size_t>(p) * BHN + static_cast<size_t>(bh) * prm.N + q_row;
      uint4* dst = reinterpret_cast<uint4*>(o_part + r * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + lane_off + c * 32, v);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]) * inv, __uint_as_float(v[8 * i + 1]) * inv);
            u.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * inv, __uint_as_float(v[8 * i + 3]) * inv);
            u.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * inv, __uint_as_float(v[8 * i + 5]) * inv);
            u.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * inv, __uint_as_float(v[8 * i + 7]) * inv);
            dst[c * 4 + i] = u;
          }
        }
      }
      if (row_ok) prm.lse_part[r] = (m + fast_log2(l)) * kLn2;
    };

    float m = -INFINITY, l = 0.0f;
    int j = 0, prev = -1;
    bool ok = true;
    const float sl2 = prm.scale_log2;
    for (int p = next_part(t, qg, 0); ok && p < t.P; p = next_part(t, qg, p + 1)) {
      const int k0 = t.part_off[p], k1 = t.part_off[p + 1];
      for (int key = k0; key < k1; key += kBN, ++j) {
        if (!mbar_wait(bar(L::S_FULL), j & 1, abort_flag, status)) { ok = false; break; }
        tc_fence_after();
        float x[kBN];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS + lane_off + 0, r0);
          tmem_ld32(tS + lane_off + 32, r1);
          tmem_ld32(tS + lane_off + 64, r2);
          tmem_ld32(tS + lane_off + 96, r3);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = __uint_as_float(r0[i]);
            x[32 + i] = __uint_as_float(r1[i]);
            x[64 + i] = __uint_as_float(r2[i]);
            x[96 + i] = __uint_as_float(r3[i]);
          }
        }
        const int nvalid = min(kBN, k1 - key);
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          x[c] = c < nvalid ? x[c] * sl2 : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
        // PV(j-1) must be complete before O is rescaled or read and before P is rewritten.
        if (j > 0) {
          if (!mbar_wait(bar(L::O_DONE), (j - 1) & 1, abort_flag, status)) { ok = false; break; }
          tc_fence_after();
        }
        if (key == k0) {
          if (prev >= 0) epilogue(prev, m, l);
          m = mt;
          l = 0.0f;
        } else {
          const float m_new = fmaxf(m, mt);
          const float alpha = fast_exp2(m - m_new);
          if (__any_sync(0xffffffffu, m_new > m)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t v[32];
              tmem_ld32(tO + lane_off + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(tO + lane_off + c * 32, v);
            }
            tmem_wait_st();
          }
          l *= alpha;
          m = m_new;
        }
        float rs = 0.0f;
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          x[c] = fast_exp2(x[c] - m);
          rs += x[c];
        }
        l += rs;
        // P row -> shared memory, K-major with the 128-byte swizzle (16-byte chunk index
        // XOR row % 8 inside each 1024-byte group of 8 rows).
#pragma unroll
        for (int ch = 0; ch < kBN / 8; ++ch) {
          const uint32_t addr = sP + (ch >> 3) * kAtomBytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
          const uint32_t w0 = pack_bf16x2(x[ch * 8 + 0], x[ch * 8 + 1]);
          const uint32_t w1 = pack_bf16x2(x[ch * 8 + 2], x[ch * 8 + 3]);
          const uint32_t w2 = pack_bf16x2(x[ch * 8 + 4], x[ch * 8 + 5]);
          const uint32_t w3 = pack_bf16x2(x[ch * 8 + 6], x[ch * 8 + 7]);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1),
                       "r"(w2), "r"(w3)
                       : "memory");
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(L::P_FULL));
        prev = p;
      }
    }
    if (ok && j > 0 && mbar_wait(bar(L::O_DONE), (j - 1) & 1, abort_flag, status)) {
      tc_fence_after();
      epilogue(prev, m, l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
int launch_impl(const TcParams& prm, int units, cudaStream_t st) {
  const int smem = Layout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  attn_tc_kernel<D><<<units, kThreads, smem, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_attn_tc(const TcParams& prm, int units, cudaStream_t st) {
  return prm.D == 64 ? launch_impl<64>(prm, units, st) : launch_impl<128>(prm, units, st);
}

int attn_tc_tile_rows() { return kBM; }

}  // namespace pa
