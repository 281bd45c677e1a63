// attn_tc.cu -- bf16 partition attention on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every (query tile, KV partition) pair selected as fresh, the attention
// state of the partition: LSE_p(i) = ln sum_j exp(s_ij) and
// O_p(i) = sum_j exp(s_ij - LSE_p(i)) v_j over the partition's valid keys, s = scale*q.k.
// This is the per-partition state of the DiTango web summary (Methodology 2, "State
// Composition"; the ring-based group state computation iterates partitions the same way).
//
// One CTA owns two 128-row query tiles (a, b) of one (batch, head) and query group and
// walks every fresh KV partition of the group in order; each K/V tile is loaded once for
// both query tiles.  The running softmax restarts at each partition boundary, where the
// epilogue writes (O_p, LSE_p).
//
// Roles (512 threads = 4 warpgroups, one CTA per SM, all 512 TMEM columns).  Launched at
// 128 registers per thread; warpgroup 0 drops to 88, the epilogue warpgroup to 72 and the
// two softmax warpgroups rise to 176 (88 + 72 + 2 * 176 = 4 * 128: the split uses exactly
// the launch allocation).
//   warp 0      TMA producer: Q_a and Q_b once, then K and V tiles of 128 keys into a
//               2-stage ring.
//   warp 1      TMEM owner and MMA issuer.  Order per KV tile j:
//                 PV_a(j), S_a(j+1), PV_b(j), S_b(j+1)
//               so that while one softmax warpgroup works on its scores the tensor pipe
//               runs the other tile's products (ping-pong).
//   warps 2, 3  idle.
//   warps 4..7  softmax of tile a; warps 8..11 softmax of tile b.  One query row per
//               thread (TMEM lane = row).  S (fp32) is read from TMEM, keys past the
//               partition end are masked, the running max is kept in the log2 domain and
//               only moved (with a rescale of O in TMEM) when it grows by more than 8
//               (2^8 bounds P), P is rounded to bf16 and written back over S in TMEM, and
//               the PV product reads it from there (A operand in TMEM).  At a partition's
//               last tile the row's (max, sum) go to shared memory for the epilogue.
//   warps 12..15 epilogue.  For each partition end, tile a then tile b: waits for the
//               partition's last PV product and its (max, sum), reads O out of TMEM, hands
//               O's columns back to the MMA issuer (the next partition's first PV
//               overwrites them), and writes O_p = O / sum and LSE_p.  The softmax
//               warpgroups never wait for these stores.
//
// Ordering facts the pipeline relies on: tcgen05.mma from one thread executes in issue
// order and tcgen05.commit tracks every earlier MMA of the thread.  So the completion of
// S_x(j+1) implies PV_x(j) is complete: the softmax may overwrite S_x / P_x columns and
// touch O_x after waiting only for S_x(j+1).  The first PV product of a partition
// (accumulate = 0) is issued only after the epilogue has read the previous partition's O.
//
// Exponentials run on MUFU (ex2.approx.ftz), one per score.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kBM = 128;        // query rows per tile (MMA M)
constexpr int kBN = 128;        // keys per tile (MMA N of S, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 512;
constexpr int kRegsLow = 88;      // warpgroup 0 (producer, MMA issuer)
constexpr int kRegsEpi = 72;      // warpgroup 3 (epilogue)
constexpr int kRegsHigh = 176;    // softmax warpgroups
static_assert(kRegsLow + kRegsEpi + 2 * kRegsHigh == kThreads / 128 * (65536 / kThreads),
              "register split must equal the launch allocation");
constexpr int kAtomBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16): one swizzle-128B box

template <int D>
struct Layout {
  static constexpr int kAtoms = D / 64;
  static constexpr int kTileBytes = kAtoms * kAtomBytes;   // a 128 x D bf16 tile
  static constexpr int kQ = 0;                             // Q_a, Q_b
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kML = kV + kStages * kTileBytes;     // (max, sum) per row: [tile][slot][row]
  static constexpr int kBar = kML + 2 * 2 * kBM * 8;
  // Per query tile x: S_FULL + x, P_LO + x, P_HI + x (softmax hand-offs), O_FINAL + x (the
  // partition's last PV complete), ML_FULL + 2x + slot ((max, sum) of partitions of that
  // parity written), O_FREE + x (the epilogue has read O).
  enum { Q_FULL = 0, K_FULL = 1, V_FULL = K_FULL + kStages, K_EMPTY = V_FULL + kStages,
         V_EMPTY = K_EMPTY + kStages, S_FULL = V_EMPTY + kStages, P_LO = S_FULL + 2, P_HI = P_LO + 2,
         O_FINAL = P_HI + 2, ML_FULL = O_FINAL + 2, O_FREE = ML_FULL + 4, NBAR = O_FREE + 2 };
  static constexpr int kTmemSlot = kBar + NBAR * 8;
  static constexpr int kAbort = kTmemSlot + 8;
  static constexpr int kUsed = kAbort + 8;
  static constexpr int kSmemBytes = kUsed + 1024;          // slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 512;               // S_a, S_b, O_a, O_b: 128 each
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;    // move the running max only when it grows by > 8
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Row max of 128 scores: 8 independent 3-input max chains, then a short tree.
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmax3(s[i], s[i + 8], s[i + 16]);
#pragma unroll
  for (int c = 24; c < 120; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], s[c + i], s[c + 8 + i]);
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[120 + i]);
  return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// First key row of the 128-key box loaded for the tile that starts at `key` in partition
// [k0, k1).  A partial last tile of a partition with at least 128 keys is loaded ending at
// k1 (shifted back over keys already processed, which the softmax masks), so K and V rows
// outside the partition are never read: masked keys get P = 0, and 0 * V is 0 only for
// finite V -- rows of another partition may be non-finite or, in the chunked relayout
// pipeline, still being written.  Partitions shorter than 128 keys load [k0, k0 + 128);
// the softmax zeroes the V rows past k1 in shared memory before the PV products read them.
__device__ __forceinline__ int tile_row0(int key, int k0, int k1) {
  return (key + kBN > k1 && k1 - kBN >= k0) ? k1 - kBN : key;
}


// Next partition >= from that is fresh for query group qg and holds at least one key.
__device__ __forceinline__ int next_part(const AttnTables& t, int qg, int from) {
  for (int p = from; p < t.P; ++p)
    if (fresh_bit(t.fresh_bits, qg, p) && t.part_off[p + 1] > t.part_off[p]) return p;
  return t.P;
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16; A (M x 16) is read from TMEM columns.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// S_x = Q_x K^T: D/16 MMAs of 128 x 128 x 16 (K-major operands, 128-byte swizzle; the
// k-step moves 32 bytes inside a 64-element swizzle atom, then to the next atom).  Called
// by a whole warp: operands stay warp-uniform and one elected lane issues each MMA (an
// issue path divergent on one lane costs ~50 cycles per MMA, a uniform one ~17-21).
template <int D>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t dq, uint64_t dk, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kAtomBytes + (kk & 3) * 32) >> 4);
    if (elect_one()) mma_bf16_ss(d_tmem, dq + off, dk + off, idesc, kk > 0);
    __syncwarp();
  }
}

// O_x (+)= P_x V: 8 MMAs of 128 x D x 16; P from TMEM (8 columns = 16 bf16 per k-step), V
// MN-major (a k-step of 16 keys moves 16 rows of 128 bytes).
// Half h of the keys: k-steps 4h .. 4h+3.
template <int D, int H>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t dv, uint32_t idesc,
                                         bool first) {
#pragma unroll
  for (int kk = H * 4; kk < H * 4 + 4; ++kk) {
    if (elect_one())
      mma_bf16_ts(d_tmem, p_tmem + kk * 8, dv + static_cast<uint32_t>((kk * 16 * 128) >> 4), idesc,
                  (first && kk == 0) ? 0u : 1u);
    __syncwarp();
  }
}

// Exponentials of half H of a row (columns 64H .. 64H+63), added to the row-sum chains
// and packed to bf16 pairs (32 TMEM columns).  Scale-and-shift and the sums use Blackwell's
// packed fp32x2 FMA / ADD (one instruction per pair).  Masked keys hold -inf, and MUFU's
// exp2(-inf) = 0 handles them, so one copy of the loop serves every tile.
template <int H>
__device__ __forceinline__ void exp_pack_half(const float (&s)[128], float m, float sl2, float2 (&acc)[4],
                                              uint32_t (&w)[32]) {
  const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-m, -m);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = H * 64 + 2 * i;
    const float2 a = __ffma2_rn(make_float2(s[c], s[c + 1]), scale2, neg_m2);
    const float e0 = fast_exp2(a.x), e1 = fast_exp2(a.y);
    acc[i & 3] = __fadd2_rn(acc[i & 3], make_float2(e0, e1));
    w[i] = pack_bf16x2(e0, e1);
  }
}

template <int D>
__device__ __forceinline__ void attn_tc_body(const TcParams& prm, const int unit) {
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

  // Decode the work unit: (b*H + h, query group, 256-row block of the group).
  const int bh = unit / prm.tiles_total;
  const int tix = unit - bh * prm.tiles_total;
  int qg = 0;
  while (qg + 1 < t.QG && t.tile_start[qg + 1] <= tix) ++qg;
  const int q_row0 = t.qg_row0[qg] + (tix - t.tile_start[qg]) * (2 * kBM);
  const int q_end = t.qg_row0[qg + 1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NBAR; ++i)
      mbar_init(bar(i), (i == L::O_FINAL || i == L::O_FINAL + 1) ? 1u : (i >= L::P_LO ? 128u : 1u));
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

  const uint32_t sQ = base + L::kQ;
  auto sK = [&](int s) { return base + L::kK + (uint32_t)s * L::kTileBytes; };
  auto sV = [&](int s) { return base + L::kV + (uint32_t)s * L::kTileBytes; };

  // Each register change sits inside its role's branch, so that the compiler allocates
  // every role's code under that role's own budget.
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch(&prm.tm_q);
      tma_prefetch(&prm.tm_k);
      tma_prefetch(&prm.tm_v);
      mbar_expect_tx(bar(L::Q_FULL), 2 * L::kTileBytes);
      for (int x = 0; x < 2; ++x)
        for (int a = 0; a < L::kAtoms; ++a)
          tma_load_3d(sQ + x * L::kTileBytes + a * kAtomBytes, &prm.tm_q, a * 64, q_row0 + x * kBM, bh,
                      bar(L::Q_FULL));
      int j = 0;
      bool ok = true;
      for (int p = next_part(t, qg, 0); ok && p < t.P; p = next_part(t, qg, p + 1)) {
        const int k1 = t.part_off[p + 1];
        const int k0 = t.part_off[p];
        for (int key = k0; key < k1; key += kBN, ++j) {
          const int s = j % kStages;
          const uint32_t ph = ((j / kStages) - 1) & 1;
          const int ty = tile_row0(key, k0, k1);
          // K's slot frees when both S products that read it complete, V's when both PV
          // products do: K runs a tile ahead of V.
          if (j >= kStages && !mbar_wait(bar(L::K_EMPTY + s), ph, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(L::K_FULL + s), L::kTileBytes);
          for (int a = 0; a < L::kAtoms; ++a)
            tma_load_3d(sK(s) + a * kAtomBytes, &prm.tm_k, a * 64, ty, bh, bar(L::K_FULL + s));
          if (j >= kStages && !mbar_wait(bar(L::V_EMPTY + s), ph, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(L::V_FULL + s), L::kTileBytes);
          for (int a = 0; a < L::kAtoms; ++a)
            tma_load_3d(sV(s) + a * kAtomBytes, &prm.tm_v, a * 64, ty, bh, bar(L::V_FULL + s));
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
    // Whole warp, warp-uniform control flow; one elected lane issues each MMA and commit.
    {
      constexpr uint32_t kIdS = idesc_bf16(kBM, kBN, false, false);   // Q K-major, K K-major
      constexpr uint32_t kIdPV = idesc_bf16(kBM, D, false, true);     // P (TMEM), V MN-major
      int T = 0;
      for (int p = next_part(t, qg, 0); p < t.P; p = next_part(t, qg, p + 1))
        T += (t.part_off[p + 1] - t.part_off[p] + kBN - 1) / kBN;
      // Descriptors of every operand tile, built once; a k-step only adds to the start
      // address field (bits 0-13, in 16-byte units).
      const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dq1 = smem_desc_sw128(sQ + L::kTileBytes, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sK(0), 16, 1024);
      const uint64_t dk1 = smem_desc_sw128(sK(1), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sV(0), kAtomBytes, 1024);
      const uint64_t dv1 = smem_desc_sw128(sV(1), kAtomBytes, 1024);
      auto commit = [&](int b) {
        if (elect_one()) mma_commit(bar(b));
        __syncwarp();
      };
      auto wait_p = [&](uint32_t b, uint32_t parity) { return mbar_wait_warp(b, parity, abort_flag, status); };
      bool ok = mbar_wait_warp(bar(L::Q_FULL), 0, abort_flag, status);
      int j = 0;
      if (ok && T > 0) {
        ok = mbar_wait_warp(bar(L::K_FULL + 0), 0, abort_flag, status) &&
             mbar_wait_warp(bar(L::V_FULL + 0), 0, abort_flag, status);
        if (ok) {
          tc_fence_after();
          issue_s<D>(tmem, dq0, dk0, kIdS);
          commit(L::S_FULL + 0);
          issue_s<D>(tmem + 128, dq1, dk0, kIdS);
          commit(L::S_FULL + 1);
          commit(L::K_EMPTY + 0);
        }
        int p = next_part(t, qg, 0);
        int key = t.part_off[p];
        int e = 0;                    // ordinal of partition p among the unit's partitions
        for (; ok && j < T; ++j) {
          const bool first = key == t.part_off[p];
          const bool last = key + kBN >= t.part_off[p + 1];
          // A partition's first PV overwrites O_x: the epilogue must have read the last one.
          const bool need_free = first && e > 0;
          const int s = j % kStages, s1 = (j + 1) % kStages;
          const bool more = j + 1 < T;
          const uint64_t dv = s ? dv1 : dv0;
          const uint64_t dk = s1 ? dk1 : dk0;
          // V(j) was waited for during the previous tile (or before the loop); operand
          // waits sit where products are already queued, off the hand-off path.
          if (need_free && !wait_p(bar(L::O_FREE + 0), (e - 1) & 1)) { ok = false; break; }
          if (!wait_p(bar(L::P_LO + 0), j & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D, 0>(tmem + 256, tmem, dv, kIdPV, first);
          // K(j+1) is checked while P hi is still being produced, so that PV hi and the
          // next S issue back to back once it arrives.
          if (more && !mbar_wait_warp(bar(L::K_FULL + s1), ((j + 1) / kStages) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          if (!wait_p(bar(L::P_HI + 0), j & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D, 1>(tmem + 256, tmem, dv, kIdPV, first);
          if (last) commit(L::O_FINAL + 0);
          if (more) {
            issue_s<D>(tmem, dq0, dk, kIdS);
            commit(L::S_FULL + 0);
          }
          if (need_free && !wait_p(bar(L::O_FREE + 1), (e - 1) & 1)) { ok = false; break; }
          if (!wait_p(bar(L::P_LO + 1), j & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D, 0>(tmem + 384, tmem + 128, dv, kIdPV, first);
          if (more && !mbar_wait_warp(bar(L::V_FULL + s1), ((j + 1) / kStages) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          if (!wait_p(bar(L::P_HI + 1), j & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D, 1>(tmem + 384, tmem + 128, dv, kIdPV, first);
          if (last) commit(L::O_FINAL + 1);
          commit(L::V_EMPTY + s);
          if (more) {
            issue_s<D>(tmem + 128, dq1, dk, kIdS);
            commit(L::S_FULL + 1);
            commit(L::K_EMPTY + s1);
          }
          key += kBN;
          if (last) {
            p = next_part(t, qg, p + 1);
            key = p < t.P ? t.part_off[p] : 0;
            ++e;
          }
        }
      }
      // The last commits must have arrived before the CTA may exit.
      if (lane == 0) {
        for (int jj = (j > kStages ? j - kStages : 0); jj < j; ++jj) {
          mbar_drain(bar(L::K_EMPTY + jj % kStages), (jj / kStages) & 1);
          mbar_drain(bar(L::V_EMPTY + jj % kStages), (jj / kStages) & 1);
        }
      }
    }
  }
  } else if (warp < 12) {
    // ---------------------------------------------------------------- softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int x = (warp - 4) >> 2;                 // query tile: 0 = a (warps 4-7), 1 = b
    const int wq = warp & 3;                       // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + x * 128;
    const uint32_t tO = tmem + lane_off + 256 + x * 128;
    float2* ml_slot = reinterpret_cast<float2*>(gbase + L::kML) + (x * 2) * kBM + row;

    float m = -INFINITY, l = 0.0f;   // running max (log2 units, scaled) and sum
    int j = 0, e = 0;
    bool ok = true;
    const float sl2 = prm.scale_log2;
    for (int p = next_part(t, qg, 0); ok && p < t.P; p = next_part(t, qg, p + 1)) {
      const int k0 = t.part_off[p], k1 = t.part_off[p + 1];
      for (int key = k0; key < k1; key += kBN, ++j) {
        if (!mbar_wait(bar(L::S_FULL + x), j & 1, abort_flag, status)) { ok = false; break; }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t r[2][64];
          tmem_ld64(tS, r[0]);
          tmem_ld64(tS + 64, r[1]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(r[i >> 6][i & 63]);
        }
        const int nvalid = min(kBN, k1 - key);
        if (nvalid < kBN) {
          // Keys outside [key, k1) of the loaded box: the leading ones of a shifted last
          // tile (already processed), or the trailing ones of a partition shorter than a tile.
          const int lo = tile_row0(key, k0, k1) < key ? kBN - nvalid : 0;
#pragma unroll
          for (int c = 0; c < kBN; ++c) s[c] = (c >= lo && c < lo + nvalid) ? s[c] : -INFINITY;
        }
        if (x == 0 && nvalid < kBN && tile_row0(key, k0, k1) == key) {
          // A partition shorter than a tile: the V box runs past the partition end into rows
          // that may be non-finite (another partition, or rows still being written).  Masked
          // keys have P = 0, but 0 * inf is NaN in the PV product, so tile a's warps zero
          // those V rows in shared memory before handing over P (both PV products of this
          // tile are issued after that hand-off).  A whole 128-byte row of each swizzle atom
          // is one key, so the swizzle does not matter here.
          const int st = j % kStages;
          if (!mbar_wait(bar(L::V_FULL + st), (j / kStages) & 1, abort_flag, status)) { ok = false; break; }
          if (row >= nvalid) {
#pragma unroll
            for (int a = 0; a < L::kAtoms; ++a) {
              uint4* dst = reinterpret_cast<uint4*>(gbase + L::kV + st * L::kTileBytes + a * kAtomBytes + row * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          fence_async_smem();
        }
        const float mt = row_max128(s) * sl2;
        if (key == k0) {
          m = mt;
          l = 0.0f;
        } else if (__any_sync(0xffffffffu, mt - m > kRescaleLog2)) {
          // Only rows whose own max grew past the bound move it (alpha = 1 elsewhere), so
          // a row's result never depends on which rows share its warp.
          const float m_new = mt - m > kRescaleLog2 ? mt : m;
          const float alpha = fast_exp2(m - m_new);
          // 16 columns at a time: the scores stay live here, and a narrow chunk keeps the
          // warpgroup inside its register budget (a rescale is rare; its speed hardly matters).
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t v[16];
            tmem_ld16(tO + c * 16, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st16(tO + c * 16, v);
          }
          l *= alpha;
          m = m_new;
        }
        // Exponentials, row sum (8 independent chains) and P packed to bf16 pairs, half a
        // row at a time; each half of P goes over S_x's first 64 columns and is handed to
        // the MMA issuer at once, so PV on keys 0-63 overlaps the exponentials of 64-127.
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        {
          uint32_t w[32];
          exp_pack_half<0>(s, m, sl2, acc, w);
          tmem_st32(tS + 0, w);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::P_LO + x));
        }
        {
          uint32_t w[32];
          exp_pack_half<1>(s, m, sl2, acc, w);
          tmem_st32(tS + 32, w);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::P_HI + x));
        }
        {
          const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
          const float2 a = __fadd2_rn(a01, a23);
          l += a.x + a.y;
        }
        if (key + kBN >= k1) {
          // The partition's last tile: its (max, sum) go to the epilogue through a slot of
          // the partition's parity (the slot is rewritten two partitions later, after the
          // epilogue has read it: see the ordering notes at the top).
          ml_slot[(e & 1) * kBM] = make_float2(m, l);
          mbar_arrive(bar(L::ML_FULL + 2 * x + (e & 1)));
          ++e;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const size_t BHN = static_cast<size_t>(prm.BH) * prm.N;
    __nv_bfloat16* o_part = static_cast<__nv_bfloat16*>(prm.o_part);
    const float2* ml_slot = reinterpret_cast<const float2*>(gbase + L::kML) + row;

    // Fresh partitions without keys: LSE = -inf, O = 0.
    for (int p = 0; p < t.P; ++p) {
      if (!fresh_bit(t.fresh_bits, qg, p) || t.part_off[p + 1] > t.part_off[p]) continue;
      for (int x = 0; x < 2; ++x) {
        const int q_row = q_row0 + x * kBM + row;
        if (q_row >= q_end) continue;
        const size_t r = static_cast<size_t>(p) * BHN + static_cast<size_t>(bh) * prm.N + q_row;
        uint4* dst = reinterpret_cast<uint4*>(o_part + r * D);
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        prm.lse_part[r] = -INFINITY;
      }
    }

    bool ok = true;
    int e = 0;
    for (int p = next_part(t, qg, 0); ok && p < t.P; p = next_part(t, qg, p + 1), ++e) {
      for (int x = 0; x < 2; ++x) {
        if (!mbar_wait(bar(L::O_FINAL + x), e & 1, abort_flag, status) ||
            !mbar_wait(bar(L::ML_FULL + 2 * x + (e & 1)), (e >> 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float2 ml = ml_slot[(x * 2 + (e & 1)) * kBM];
        const float inv = 1.0f / ml.y;
        const int q_row = q_row0 + x * kBM + row;
        const bool row_ok = q_row < q_end;
        const size_t r = static_cast<size_t>(p) * BHN + static_cast<size_t>(bh) * prm.N + q_row;
        uint4* dst = reinterpret_cast<uint4*>(o_part + r * D);
        const uint32_t tO = tmem + lane_off + 256 + x * 128;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
          if (c == D / 32 - 1) {
            // O_x is out of TMEM: the issuer may start the next partition's PV into it.
            tc_fence_before();
            mbar_arrive(bar(L::O_FREE + x));
          }
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
        if (row_ok) prm.lse_part[r] = (ml.x + fast_log2(ml.y)) * kLn2;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// One CTA per work unit.  Unit = blockIdx.x; or, for a grid of a few waves, the unit that
// the host's longest-first order puts at that position: the hardware hands out CTAs in
// blockIdx order as SMs free up, so the longest units start first and the last wave holds
// the shortest ones (a shorter tail when units differ in length).
template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams prm) {
  attn_tc_body<D>(prm, static_cast<int>(blockIdx.x));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_ordered_kernel(const __grid_constant__ TcParams prm,
                                                                      const __grid_constant__ TcUnitOrder ord) {
  attn_tc_body<D>(prm, static_cast<int>(ord.unit[blockIdx.x]));
}

template <int D>
int launch_impl(const TcParams& prm, const TcUnitOrder* ord, int units, cudaStream_t st) {
  const int smem = Layout<D>::kSmemBytes;
  cudaError_t e = ord ? cudaFuncSetAttribute(attn_tc_ordered_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
                      : cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (ord)
    attn_tc_ordered_kernel<D><<<units, kThreads, smem, st>>>(prm, *ord);
  else
    attn_tc_kernel<D><<<units, kThreads, smem, st>>>(prm);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_attn_tc(const TcParams& prm, const TcUnitOrder* ord, int units, cudaStream_t st) {
  return prm.D == 64 ? launch_impl<64>(prm, ord, units, st) : launch_impl<128>(prm, ord, units, st);
}

// Query rows per work unit (two 128-row tiles).
int attn_tc_tile_rows() { return 2 * kBM; }

}  // namespace pa
