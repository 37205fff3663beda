// fa_bwd_kernel.cuh -- backward pass of exact attention on sm_100a.
//
// The pages state that FlashAttention keeps no N x N matrix for the backward pass: it
// computes the attention again from Q, K, V and the saved row log-sum-exp ("Flash
// Attention" page, section "Zentrale technische Innovationen", the recomputation bullet).
// For O = P V, P = softmax(S) row by row, S = scale * Q K^T (+ causal mask) and an
// upstream gradient dO, the gradients are
//
//   P_ij  = exp(scale * q_i . k_j - LSE_i)        (recomputed from the forward's LSE)
//   dV    = P^T dO
//   dP    = dO V^T
//   dS_ij = P_ij (dP_ij - D_i),  D_i = sum_t dO_it O_it  (= sum_j P_ij dP_ij)
//   dK    = scale * dS^T Q
//   dQ    = scale * dS K
//
// Work decomposition: a unit is one block of BN = 128 keys of one (batch, K/V head); its
// CTA keeps K_j and V_j in shared memory and dK_j, dV_j in tensor memory for the whole
// unit, and walks every query head of the group and every block of BM = 64 queries (from
// the diagonal on under the causal mask).  Per step five tcgen05 MMAs:
//
//   S^T  = K_j Q_i^T      M=128 keys, N=64 queries, K=D (SS, both K-major)
//   dP^T = V_j dO_i^T     same shape
//   dQ^T = K_j^T dS^T     M=128 head dims, N=64 queries, K=128 keys (SS, both MN-major;
//                         at D = 64 the upper 64 rows of K_j^T are a tile of zeros)
//   dV  += P^T dO_i       M=128 keys, N=D, K=64 queries (A = P^T from tensor memory)
//   dK  += dS^T Q_i       same shape (A = dS^T from tensor memory)
//
// D (the head dimension) is 64 or 128.
//
// dQ^T goes from tensor memory through a shared-memory staging tile to a bulk tensor
// reduce-add (TMA) into a zeroed fp32 accumulator in global memory (each query block
// receives one contribution per key block); a last kernel scales it and rounds to bf16.  dK, dV leave once per unit, with no atomics: the group's query heads
// are summed inside the unit.
//
// Tensor memory (512 columns): S^T of step buffer b at b*128 (64 columns; after the
// softmax, P^T and dS^T as packed bf16), dP^T of buffer b at b*128 + 64 (then dQ^T of the
// same step), dV at 256, dK at 256 + D.  Two step buffers let the softmax of step i+1 run
// while the tensor core works on step i.  Q_i, dO_i and the two per-query vectors sit in a
// ring of QSTAGES shared-memory stages, so their copies run two steps ahead of the MMAs
// that read them; dS^T has one shared-memory buffer (the softmax of step g writes it once
// the dQ^T product of step g-1 has read it).
//
// Warps: 0-3 and 4-7 are the "softmax" warpgroups (thread = key row; warpgroup h takes
// queries 32h .. 32h+31 of the step, and at the end of a unit writes dV (h=0) or dK
// (h=1)); 8-11 drain dQ^T (thread = head dimension); 12 allocates tensor memory and issues
// the MMAs; 13 issues the TMA copies.  At D = 64 only drain warps 8-9 own head dims.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_fwd_kernel.cuh"  // device error word and bounded waits
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int BN = 128;                  // keys per unit (tensor-memory lanes)
constexpr int BM = 64;                   // queries per step
constexpr int NUM_THREADS = 448;         // 14 warps
constexpr int DRAIN_WARP0 = 8;
constexpr int MMA_WARP = 12;
constexpr int TMA_WARP = 13;
constexpr int KV_BOX = BN * 128;         // one 128-byte-wide TMA box of a K or V tile (16 KB)
constexpr int Q_BOX = BM * 128;          // one box of a Q or dO tile (8 KB)
constexpr int DS_TILE = BN * BM * 2;     // dS^T [keys][queries] bf16, 128-byte rows: 16 KB
constexpr int VEC_BYTES = 2 * BM * 4;    // per step: LSE*log2(e) and D for BM queries
constexpr int QSTAGES = 3;               // ring of Q, dO and vector stages
constexpr int DQ_STAGE = 32 * BM * 4;    // per drain warp: 64 queries x 32 head dims fp32
constexpr int NUM_BARS = 2 + 2 * QSTAGES + 2 * 4 + 3 + 2 * UNIT_RING;

// Tensor-memory columns of the step buffers.
__host__ __device__ constexpr uint32_t s_col(int b) { return b * 128; }
__host__ __device__ constexpr uint32_t dp_col(int b) { return b * 128 + 64; }

// Head-dimension-dependent layout (D = 64 or 128).  The dQ^T product always has M = 128
// head-dimension rows: at D = 64 the second 64 rows of its A operand (K^T) come from a
// 16 KB tile of zeros, so rows 64..127 of dQ^T are zero and are not reduced.  That costs
// half a product per step and keeps the tensor-memory lane layout of M = 128.
template <int D>
struct BCfg {
  static_assert(D == 64 || D == 128, "head dims of the backward kernel");
  static constexpr int NBOX = D * 2 / 128;             // 128-byte boxes per row
  static constexpr int KV_TILE = NBOX * KV_BOX;
  static constexpr int Q_TILE = NBOX * Q_BOX;
  static constexpr int DRAIN_WARPS = D / 32;           // drain warps that own head dims
  // Shared memory map (offsets from a 1024-aligned base).
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KV_TILE;
  static constexpr int Z_OFF = V_OFF + KV_TILE;
  static constexpr int Z_BYTES = D < 128 ? KV_BOX : 0;
  static constexpr int Q_OFF = Z_OFF + Z_BYTES;
  static constexpr int DO_OFF = Q_OFF + QSTAGES * Q_TILE;
  static constexpr int DS_OFF = DO_OFF + QSTAGES * Q_TILE;
  static constexpr int DQS_OFF = DS_OFF + DS_TILE;
  static constexpr int VEC_OFF = DQS_OFF + DRAIN_WARPS * DQ_STAGE;
  static constexpr int BAR_OFF = VEC_OFF + QSTAGES * VEC_BYTES;
  static constexpr int CTL_OFF = BAR_OFF + NUM_BARS * 8;
  // control words: TMEM base, abort flag, 2 spare, then the ring of published units
  static constexpr int SMEM_BYTES = 1024 + CTL_OFF + 16 + 4 * UNIT_RING;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // Tensor memory: step buffers at 0..255, dV at 256, dK after it.
  static constexpr uint32_t DV_COL = 256, DK_COL = 256 + D;
  static constexpr uint32_t IDESC_S = ptx::make_idesc(1, BN, BM, 0);        // S^T, dP^T
  static constexpr uint32_t IDESC_ACC = ptx::make_idesc(1, BN, D, 1);       // dV, dK
  static constexpr uint32_t IDESC_DQ = ptx::make_idesc_ab(1, 128, BM, 1, 1);  // dQ^T
  // leading-byte offset of the K^T operand: from head dims 0..63 to 64..127
  static constexpr uint32_t KT_LBO = D == 128 ? KV_BOX : Z_OFF - K_OFF;
};

constexpr uint32_t ERR_WAIT_BWD = 1u << 6;

struct BwdParams {
  const float *l2;     // [B*Hq, Npad]: LSE * log2(e), +inf past Nq
  const float *dd;     // [B*Hq, Npad]: D = rowsum(dO o O), 0 past Nq
  uint16_t *dk, *dv;   // bf16 [B*Hkv, Nk, D]
  int B, Hq, Hkv, Nq, Nk, Npad, group;
  int diag;            // Nk - Nq: the causal mask admits key j for query i iff j <= i + diag
  int num_kb;          // ceil(Nk / BN)
  int num_qb;          // ceil(Nq / BM)
  int num_units;       // B * Hkv * num_kb
  unsigned int *sched; // this launch's work counters (see g_fa_sched)
  float scale_log2;    // scale * log2(e)
  float scale;
};

struct BUnit {
  int bhk;    // b * Hkv + hk
  int b, hk;
  int j;      // key block
  int i0;     // first query block visited
  int nq;     // query blocks visited per query head
  int steps;  // group * nq
};

template <bool CAUSAL>
__device__ __forceinline__ BUnit decode_unit(const BwdParams &p, int u) {
  BUnit w;
  w.bhk = u / p.num_kb;
  w.j = u % p.num_kb;
  w.b = w.bhk / p.Hkv;
  w.hk = w.bhk % p.Hkv;
  // Under the causal mask query i sees key j only if j <= i + diag: blocks of queries that
  // end before the key block's first admitting query are skipped.  Query Nq - 1 admits
  // every key, so no unit is left without steps.
  const int first = w.j * BN - p.diag;  // first query that sees key j*BN
  w.i0 = CAUSAL && first > 0 ? first / BM : 0;
  w.nq = p.num_qb - w.i0;
  w.steps = p.group * w.nq;
  return w;
}

// (query head row index b*Hq + hq, query block) of step s of unit w.
__device__ __forceinline__ void step_coords(const BwdParams &p, const BUnit &w, int s, int &bh,
                                            int &i) {
  bh = w.b * p.Hq + w.hk * p.group + s / w.nq;
  i = w.i0 + s % w.nq;
}

struct BBars {
  uint32_t base;
  __device__ uint32_t kv_full() const { return base; }
  __device__ uint32_t kv_empty() const { return base + 8u; }
  __device__ uint32_t q_full(int st) const { return base + 8u * (2 + st); }
  __device__ uint32_t q_empty(int st) const { return base + 8u * (2 + QSTAGES + st); }
  static constexpr int B0 = 2 + 2 * QSTAGES;
  __device__ uint32_t sdp_full(int b) const { return base + 8u * (B0 + b); }
  __device__ uint32_t ds_full(int b) const { return base + 8u * (B0 + 2 + b); }
  __device__ uint32_t dq_full(int b) const { return base + 8u * (B0 + 4 + b); }
  __device__ uint32_t dq_empty(int b) const { return base + 8u * (B0 + 6 + b); }
  __device__ uint32_t acc_full() const { return base + 8u * (B0 + 8); }
  __device__ uint32_t acc_empty() const { return base + 8u * (B0 + 9); }
  __device__ uint32_t drain() const { return base + 8u * (B0 + 10); }
  // ring of published work units (TMA warp -> MMA, softmax and dQ warps)
  __device__ uint32_t unit_full(int s) const { return base + 8u * (B0 + 11 + s); }
  __device__ uint32_t unit_empty(int s) const { return base + 8u * (B0 + 11 + UNIT_RING + s); }
};

// ---------------------------------------------------------------------------- producer

template <int D, bool CAUSAL>
__device__ void load_role(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                          const CUtensorMap *tmDO, const BwdParams &p, uint32_t smem,
                          const BBars &bar, volatile uint32_t *unit_ring,
                          volatile uint32_t *abort_flag) {
  using C = BCfg<D>;
  ptx::prefetch_tmap(tmQ);
  ptx::prefetch_tmap(tmK);
  ptx::prefetch_tmap(tmV);
  ptx::prefetch_tmap(tmDO);
  uint32_t units_issued = 0, steps_issued = 0, published = 0;
  const uint32_t num_units = static_cast<uint32_t>(p.num_units);
  // first unit blockIdx.x, then units claimed from the launch's counter (see the forward)
  for (uint32_t u = blockIdx.x;; u = gridDim.x + atomicAdd(p.sched, 1u)) {
    {  // publish u (or, past the last unit, the end of the list)
      const int s = published % UNIT_RING;
      if (!wait_phase(bar.unit_empty(s), ((published / UNIT_RING) & 1u) ^ 1u, abort_flag,
                      ERR_WAIT_BWD))
        goto drain;
      unit_ring[s] = u;
      ptx::mbar_arrive(bar.unit_full(s));
      ++published;
    }
    if (u >= num_units) break;
    const BUnit w = decode_unit<CAUSAL>(p, static_cast<int>(u));
    if (!wait_phase(bar.kv_empty(), (units_issued & 1u) ^ 1u, abort_flag, ERR_WAIT_BWD))
      goto drain;
    ptx::mbar_arrive_expect_tx(bar.kv_full(), 2 * C::KV_TILE);
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx) {
      ptx::tma_load_3d(smem + C::K_OFF + bx * KV_BOX, tmK, bar.kv_full(), bx * 64, w.j * BN, w.bhk);
      ptx::tma_load_3d(smem + C::V_OFF + bx * KV_BOX, tmV, bar.kv_full(), bx * 64, w.j * BN, w.bhk);
    }
    ++units_issued;
    for (int s = 0; s < w.steps; ++s) {
      const int st = steps_issued % QSTAGES;
      const uint32_t use = steps_issued / QSTAGES;
      if (!wait_phase(bar.q_empty(st), (use & 1u) ^ 1u, abort_flag, ERR_WAIT_BWD)) goto drain;
      int bh, i;
      step_coords(p, w, s, bh, i);
      ptx::mbar_arrive_expect_tx(bar.q_full(st), 2 * C::Q_TILE + VEC_BYTES);
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx) {
        ptx::tma_load_3d(smem + C::Q_OFF + st * C::Q_TILE + bx * Q_BOX, tmQ, bar.q_full(st), bx * 64,
                         i * BM, bh);
        ptx::tma_load_3d(smem + C::DO_OFF + st * C::Q_TILE + bx * Q_BOX, tmDO, bar.q_full(st),
                         bx * 64, i * BM, bh);
      }
      const long long voff = static_cast<long long>(bh) * p.Npad + i * BM;
      ptx::bulk_load(smem + C::VEC_OFF + st * VEC_BYTES, p.l2 + voff, BM * 4, bar.q_full(st));
      ptx::bulk_load(smem + C::VEC_OFF + st * VEC_BYTES + BM * 4, p.dd + voff, BM * 4,
                     bar.q_full(st));
      ++steps_issued;
    }
  }
drain:
  // Let every copy this thread started land before the CTA exits (immediate on the normal
  // path, where the consumers have already waited for them).
  if (units_issued > 0) drain_wait(bar.kv_full(), (units_issued - 1) & 1u);
  for (uint32_t st = 0; st < QSTAGES; ++st)
    if (steps_issued > st) {
      const uint32_t last = st + QSTAGES * ((steps_issued - 1 - st) / QSTAGES);
      drain_wait(bar.q_full(st), (last / QSTAGES) & 1u);
    }
}

// ---------------------------------------------------------------------------- MMA issuer

// S^T or dP^T: A = K_j or V_j (128 rows, D/64 128-byte column boxes, K-major), B = Q_i or
// dO_i (64 rows, same boxes, K-major); K = D head dims in steps of 16.
template <int D>
__device__ __forceinline__ void issue_sdp(uint32_t tmem_d, uint64_t a_desc, uint64_t b_desc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    constexpr uint32_t step = 32;  // bytes along the head dim per MMA
    const uint32_t kb = kk * step;
    const uint32_t aoff = ((kb / 128) * KV_BOX + (kb % 128)) >> 4;
    const uint32_t boff = ((kb / 128) * Q_BOX + (kb % 128)) >> 4;
    ptx::mma_bf16_ss_elect(tmem_d, a_desc + aoff, b_desc + boff, BCfg<D>::IDESC_S,
                           kk > 0 ? 1u : 0u);
  }
}

// dV += P^T dO_i or dK += dS^T Q_i: A from tensor memory (keys x 64 queries as packed
// bf16; queries 0-31 at columns 0-15 (+16 for dS), queries 32-63 at 32-47), B = dO_i or
// Q_i read MN-major (64 query rows of 128-byte head-dim boxes); K = 64 queries in steps
// of 16 (8 packed columns, 16 rows of 128 bytes).
template <int D>
__device__ __forceinline__ void issue_acc(uint32_t tmem_d, uint32_t tmem_a, uint64_t b_desc,
                                          uint32_t accumulate) {
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk) {
    const uint32_t a = tmem_a + (kk / 2) * 32 + (kk % 2) * 8;
    const uint32_t boff = (kk * 16 * 128) >> 4;
    ptx::mma_bf16_ts_elect(tmem_d, a, b_desc + boff, BCfg<D>::IDESC_ACC,
                           kk > 0 ? 1u : accumulate);
  }
}

// dQ^T = K_j^T dS^T: A = K_j read MN-major (M = 128 head dims: two boxes KT_LBO apart, the
// second a tile of zeros at D = 64), B = dS^T
// read MN-major (N = 64 queries in one 128-byte row); K = 128 keys in steps of 16 rows.
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t tmem_d, uint64_t a_desc, uint64_t b_desc) {
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    const uint32_t off = (kk * 16 * 128) >> 4;
    ptx::mma_bf16_ss_elect(tmem_d, a_desc + off, b_desc + off, BCfg<D>::IDESC_DQ,
                           kk > 0 ? 1u : 0u);
  }
}

template <int D, bool CAUSAL>
__device__ void mma_role(const BwdParams &p, uint32_t smem, uint32_t tmem, const BBars &bar,
                         volatile uint32_t *unit_ring, volatile uint32_t *abort_flag) {
  using C = BCfg<D>;
  const uint64_t k_a = ptx::smem_desc_sw128(smem + C::K_OFF, 16, 1024);
  const uint64_t v_a = ptx::smem_desc_sw128(smem + C::V_OFF, 16, 1024);
  const uint64_t k_t = ptx::smem_desc_sw128(smem + C::K_OFF, C::KT_LBO, 1024);
  auto wait = [&](uint32_t b, uint32_t parity) {
    const bool ok = wait_phase(b, parity, abort_flag, ERR_WAIT_BWD);
    return __all_sync(0xffffffffu, ok);
  };
  // S^T and dP^T of global step g (buffer g & 1).
  auto start_step = [&](uint32_t g) {
    const int b = g & 1u, st = g % QSTAGES;
    const uint32_t use = g >> 1;
    if (!wait(bar.q_full(st), (g / QSTAGES) & 1u)) return false;
    ptx::tc_fence_after();
    issue_sdp<D>(tmem + s_col(b), k_a, ptx::smem_desc_sw128(smem + C::Q_OFF + st * C::Q_TILE, 16, 1024));
    // dP^T lands where dQ^T of this buffer's previous step was: wait for its drain.
    if (!wait(bar.dq_empty(b), (use & 1u) ^ 1u)) return false;
    ptx::tc_fence_after();
    issue_sdp<D>(tmem + dp_col(b), v_a,
              ptx::smem_desc_sw128(smem + C::DO_OFF + st * C::Q_TILE, 16, 1024));
    ptx::mma_commit_elect(bar.sdp_full(b));
    return true;
  };
  uint32_t gm = 0, unit_it = 0, taken = 0;
  bool ok = true;
  for (; ok; ++unit_it) {
    uint32_t u;
    if (!take_unit(bar, unit_ring, taken, abort_flag, ERR_WAIT_BWD, u) ||
        u >= static_cast<uint32_t>(p.num_units))
      break;
    const BUnit w = decode_unit<CAUSAL>(p, static_cast<int>(u));
    if (!wait(bar.kv_full(), unit_it & 1u)) break;
    ptx::tc_fence_after();
    for (int s = 0; s < 2 && s < w.steps && ok; ++s) ok = start_step(gm + s);
    for (int s = 0; s < w.steps && ok; ++s) {
      const uint32_t g = gm + s;
      const int b = g & 1u, st = g % QSTAGES;
      const uint32_t use = g >> 1;
      if (!(ok = wait(bar.ds_full(b), use & 1u))) break;
      ptx::tc_fence_after();
      issue_dq<D>(tmem + dp_col(b), k_t, ptx::smem_desc_sw128(smem + C::DS_OFF, DS_TILE, 1024));
      ptx::mma_commit_elect(bar.dq_full(b));
      if (s == 0) {
        if (!(ok = wait(bar.acc_empty(), (unit_it & 1u) ^ 1u))) break;
        ptx::tc_fence_after();
      }
      issue_acc<D>(tmem + C::DV_COL, tmem + s_col(b),
                ptx::smem_desc_sw128(smem + C::DO_OFF + st * C::Q_TILE, Q_BOX, 1024), s > 0 ? 1u : 0u);
      issue_acc<D>(tmem + C::DK_COL, tmem + s_col(b) + 16,
                ptx::smem_desc_sw128(smem + C::Q_OFF + st * C::Q_TILE, Q_BOX, 1024), s > 0 ? 1u : 0u);
      ptx::mma_commit_elect(bar.q_empty(st));
      if (s == w.steps - 1) {
        ptx::mma_commit_elect(bar.acc_full());
        ptx::mma_commit_elect(bar.kv_empty());
      }
      if (s + 2 < w.steps) ok = start_step(g + 2);
    }
    gm += w.steps;
  }
  // Wait until every MMA issued by this warp has finished before tensor memory is freed.
  ptx::mma_commit_elect(bar.drain());
  drain_wait(bar.drain(), 0);
}

// ---------------------------------------------------------------------------- softmax

// Recompute P^T and form dS^T for one step: this thread owns key row `key` and queries
// q0 .. q0+31 (q0 = i*BM + 32h).  Writes P^T and dS^T as packed bf16 into its own 32
// columns of the S^T buffer and dS^T into the shared-memory tile (128-byte swizzle: the
// 16-byte chunk c of row r sits at chunk c ^ (r % 8)).
template <int D, bool CAUSAL>
__device__ __forceinline__ bool softmax_step(const BwdParams &p, uint32_t tmem_row, uint32_t smem,
                                             const BBars &bar, uint32_t g, int h, int row,
                                             int key, int q0, bool need_mask,
                                             volatile uint32_t *abort_flag) {
  using C = BCfg<D>;
  const int b = g & 1u, st = g % QSTAGES;
  uint32_t sr[2][16], dr[2][16];
  ptx::tmem_ld16(tmem_row + s_col(b) + h * 32, sr[0]);
  ptx::tmem_ld16(tmem_row + s_col(b) + h * 32 + 16, sr[1]);
  ptx::tmem_ld16(tmem_row + dp_col(b) + h * 32, dr[0]);
  ptx::tmem_ld16(tmem_row + dp_col(b) + h * 32 + 16, dr[1]);
  ptx::tmem_wait_ld();
  ptx::reg_fence16(sr[0]);
  ptx::reg_fence16(sr[1]);
  ptx::reg_fence16(dr[0]);
  ptx::reg_fence16(dr[1]);
  const float *vec = reinterpret_cast<const float *>(
      __cvta_shared_to_generic(smem + C::VEC_OFF + st * VEC_BYTES));
  const float4 *l2v = reinterpret_cast<const float4 *>(vec + h * 32);
  const float4 *ddv = reinterpret_cast<const float4 *>(vec + BM + h * 32);
  uint32_t pp[16], pd[16];
#pragma unroll
  for (int c4 = 0; c4 < 8; ++c4) {
    const float4 l4 = l2v[c4], d4 = ddv[c4];
    const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
    float pv[4], sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c4 * 4 + e;
      const float s = __uint_as_float(sr[c / 16][c % 16]);
      const float dpv = __uint_as_float(dr[c / 16][c % 16]);
      float pe = ptx::ex2(fmaf(s, p.scale_log2, -lv[e]));
      if (need_mask && (key >= p.Nk || (CAUSAL && key > q0 + c + p.diag))) pe = 0.f;
      pv[e] = pe;
      sv[e] = pe * (dpv - dv[e]);
    }
    pp[c4 * 2] = ptx::pack_bf16x2(pv[0], pv[1]);
    pp[c4 * 2 + 1] = ptx::pack_bf16x2(pv[2], pv[3]);
    pd[c4 * 2] = ptx::pack_bf16x2(sv[0], sv[1]);
    pd[c4 * 2 + 1] = ptx::pack_bf16x2(sv[2], sv[3]);
  }
  ptx::tmem_st16(tmem_row + s_col(b) + h * 32, pp);
  ptx::tmem_st16(tmem_row + s_col(b) + h * 32 + 16, pd);
  // the single dS^T buffer is free once the dQ^T product of the previous step has run
  if (g > 0 && !wait_phase(bar.dq_full((g - 1) & 1u), ((g - 1) >> 1) & 1u, abort_flag,
                           ERR_WAIT_BWD))
    return false;
  const uint32_t ds_row = smem + C::DS_OFF + row * 128;
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const uint32_t chunk = static_cast<uint32_t>(h * 4 + cc) ^ static_cast<uint32_t>(row & 7);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ds_row + chunk * 16),
                 "r"(pd[cc * 4]), "r"(pd[cc * 4 + 1]), "r"(pd[cc * 4 + 2]), "r"(pd[cc * 4 + 3])
                 : "memory");
  }
  ptx::tmem_wait_st();
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  return true;
}

template <int D, bool CAUSAL>
__device__ void softmax_role(const BwdParams &p, uint32_t smem, uint32_t tmem, const BBars &bar,
                             volatile uint32_t *unit_ring, volatile uint32_t *abort_flag) {
  using C = BCfg<D>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = warp / 4;                     // query half of the step
  const int row = (warp % 4) * 32 + lane;     // key row within the block
  const uint32_t tmem_row = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
  uint32_t gs = 0, unit_it = 0, taken = 0;
  for (;; ++unit_it) {
    uint32_t u;
    if (!take_unit(bar, unit_ring, taken, abort_flag, ERR_WAIT_BWD, u) ||
        u >= static_cast<uint32_t>(p.num_units))
      return;
    const BUnit w = decode_unit<CAUSAL>(p, static_cast<int>(u));
    const int key = w.j * BN + row;
    for (int s = 0; s < w.steps; ++s) {
      const uint32_t g = gs + s;
      const int b = g & 1u;
      if (!wait_phase(bar.sdp_full(b), (g >> 1) & 1u, abort_flag, ERR_WAIT_BWD)) return;
      ptx::tc_fence_after();
      int bh, i;
      step_coords(p, w, s, bh, i);
      const int q0 = i * BM + h * 32;
      // masking is needed on the key tail block and, causally, where the first query of
      // the block does not admit the block's last key (this covers the rows that admit
      // no key at all when Nq > Nk: their LSE is -inf and only the mask zeroes P)
      const bool need_mask =
          (w.j * BN + BN > p.Nk) || (CAUSAL && q0 + p.diag < w.j * BN + BN - 1);
      if (!softmax_step<D, CAUSAL>(p, tmem_row, smem, bar, g, h, row, key, q0, need_mask,
                                abort_flag))
        return;
      ptx::mbar_arrive(bar.ds_full(b));
    }
    gs += w.steps;
    // Unit epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK, as bf16 rows.
    if (!wait_phase(bar.acc_full(), unit_it & 1u, abort_flag, ERR_WAIT_BWD)) return;
    ptx::tc_fence_after();
    const float mult = h == 0 ? 1.f : p.scale;
    uint16_t *out = (h == 0 ? p.dv : p.dk) + (static_cast<long long>(w.bhk) * p.Nk + key) * D;
#pragma unroll 1
    for (int c = 0; c < D / 16; ++c) {
      uint32_t r[16];
      ptx::tmem_ld16(tmem_row + (h == 0 ? C::DV_COL : C::DK_COL) + c * 16, r);
      ptx::tmem_wait_ld();
      ptx::reg_fence16(r);
      uint32_t o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        o[e] = ptx::pack_bf16x2(__uint_as_float(r[2 * e]) * mult,
                                __uint_as_float(r[2 * e + 1]) * mult);
      if (key < p.Nk) {
        uint4 *dst = reinterpret_cast<uint4 *>(out + c * 16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar.acc_empty());
  }
}

// ---------------------------------------------------------------------------- dQ drain

// Thread = head dimension t (warp w of the group owns t = 32w .. 32w+31): after each
// step's dQ^T lands, read its 64 query columns, write them as a [64 queries][32 dims]
// fp32 tile into the warp's staging buffer (one 128-byte row per query, so every store
// instruction of the warp fills one row) and add the tile into the accumulator with one
// bulk tensor reduce-add.  Queries past Nq fall outside the tensor and are not written.
template <int D, bool CAUSAL>
__device__ void dq_role(const CUtensorMap *tmDQ, const BwdParams &p, uint32_t smem, uint32_t tmem,
                        const BBars &bar, volatile uint32_t *unit_ring,
                        volatile uint32_t *abort_flag) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wq = warp % 4;
  const uint32_t tmem_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  using C = BCfg<D>;
  // warps whose head dims lie past D (D = 64: the zero rows of dQ^T) read and release
  // the buffer but add nothing
  const bool owner = wq < C::DRAIN_WARPS;
  const uint32_t stage = smem + C::DQS_OFF + (owner ? wq : 0) * DQ_STAGE;
  if (lane == 0) ptx::prefetch_tmap(tmDQ);
  uint32_t gd = 0, taken = 0;
  bool pending = false;
  for (;;) {
    uint32_t u;
    if (!take_unit(bar, unit_ring, taken, abort_flag, ERR_WAIT_BWD, u) ||
        u >= static_cast<uint32_t>(p.num_units))
      break;
    const BUnit w = decode_unit<CAUSAL>(p, static_cast<int>(u));
    for (int s = 0; s < w.steps; ++s) {
      const uint32_t g = gd + s;
      const int b = g & 1u;
      const bool ok = wait_phase(bar.dq_full(b), (g >> 1) & 1u, abort_flag, ERR_WAIT_BWD);
      if (!__all_sync(0xffffffffu, ok)) goto done;
      ptx::tc_fence_after();
      uint32_t r[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld16(tmem_row + dp_col(b) + c * 16, r[c]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::reg_fence16(r[c]);
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar.dq_empty(b));
      if (!owner) continue;
      // the previous reduce must have read the staging tile before it is overwritten
      if (pending && lane == 0) ptx::bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < BM; ++c)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage + c * 128 + lane * 4),
                     "r"(r[c / 16][c % 16])
                     : "memory");
      ptx::fence_proxy_async_smem();
      __syncwarp();
      int bh, i;
      step_coords(p, w, s, bh, i);
      if (lane == 0) {
        ptx::tma_reduce_add_3d(tmDQ, stage, wq * 32, i * BM, bh);
        ptx::bulk_commit_group();
      }
      pending = true;
    }
    gd += w.steps;
  }
done:
  // every reduce must be complete before the CTA exits
  if (lane == 0) ptx::bulk_wait_all();
  __syncwarp();
}

// ---------------------------------------------------------------------------- kernels

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t smem = (raw + 1023u) & ~1023u;  // 1024-aligned for 128-byte swizzle
  uint8_t *smem_gen = smem_raw + (smem - raw);
  const BBars bar{smem + C::BAR_OFF};
  uint32_t *ctl = reinterpret_cast<uint32_t *>(smem_gen + C::CTL_OFF);
  volatile uint32_t *tmem_slot = ctl;
  volatile uint32_t *abort_flag = ctl + 1;
  volatile uint32_t *unit_ring = ctl + 4;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar.kv_full(), 1);
    ptx::mbar_init(bar.kv_empty(), 1);
    for (int st = 0; st < QSTAGES; ++st) {
      ptx::mbar_init(bar.q_full(st), 1);
      ptx::mbar_init(bar.q_empty(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar.sdp_full(b), 1);
      ptx::mbar_init(bar.ds_full(b), 256);
      ptx::mbar_init(bar.dq_full(b), 1);
      ptx::mbar_init(bar.dq_empty(b), 128);
    }
    ptx::mbar_init(bar.acc_full(), 1);
    ptx::mbar_init(bar.acc_empty(), 256);
    ptx::mbar_init(bar.drain(), 1);
    for (int s = 0; s < UNIT_RING; ++s) {
      ptx::mbar_init(bar.unit_full(s), 1);
      ptx::mbar_init(bar.unit_empty(s), 13);  // MMA warp, 8 softmax warps, 4 dQ warps
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    ptx::tmem_alloc(ptx::smem_addr(ctl), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (C::Z_BYTES > 0) {
    // the zero rows of the K^T operand (D = 64), visible to the tensor core
    for (int o = threadIdx.x * 16; o < C::Z_BYTES; o += NUM_THREADS * 16)
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(smem + C::Z_OFF + o), "r"(0u)
                   : "memory");
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < DRAIN_WARP0) {
    softmax_role<D, CAUSAL>(p, smem, tmem, bar, unit_ring, abort_flag);
  } else if (warp < MMA_WARP) {
    dq_role<D, CAUSAL>(&tmDQ, p, smem, tmem, bar, unit_ring, abort_flag);
  } else if (warp == MMA_WARP) {
    mma_role<D, CAUSAL>(p, smem, tmem, bar, unit_ring, abort_flag);
    __syncwarp();
  } else if (warp == TMA_WARP) {
    if (lane == 0)
      load_role<D, CAUSAL>(&tmQ, &tmK, &tmV, &tmDO, p, smem, bar, unit_ring, abort_flag);
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
  // every claim of this CTA is done: count the CTA out; the last one resets the counters
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
  }
}

// Per query row: D = sum_t dO_t O_t (fp32 from bf16) and LSE * log2(e), into arrays
// padded to Npad rows per (batch, head) (D = 0, LSE = +inf on the padding, so padded
// queries contribute nothing).  One warp per row, HD / 32 elements per lane.
template <int HD>
__global__ void fa_bwd_prep_kernel(const uint16_t *__restrict__ o, const uint16_t *__restrict__ dout,
                                   const float *__restrict__ lse, float *__restrict__ l2,
                                   float *__restrict__ dd, long long rows_padded, int Nq, int Npad) {
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (r >= rows_padded) return;
  const long long bh = r / Npad;
  const int q = static_cast<int>(r - bh * Npad);
  if (q >= Nq) {
    if (lane == 0) {
      l2[r] = __int_as_float(0x7f800000);
      dd[r] = 0.f;
    }
    return;
  }
  const long long row = bh * Nq + q;
  constexpr int W = HD / 64;  // 32-bit words (bf16 pairs) per lane
  const uint32_t *a = reinterpret_cast<const uint32_t *>(o + row * HD) + lane * W;
  const uint32_t *g = reinterpret_cast<const uint32_t *>(dout + row * HD) + lane * W;
  float s = 0.f;
#pragma unroll
  for (int n = 0; n < W; ++n) {
    s += __uint_as_float(a[n] << 16) * __uint_as_float(g[n] << 16);
    s += __uint_as_float(a[n] & 0xffff0000u) * __uint_as_float(g[n] & 0xffff0000u);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    dd[r] = s;
    l2[r] = lse[row] * 1.4426950408889634f;
  }
}

// dQ = scale * dq_acc, rounded to bf16; 4 elements per thread.
__global__ void fa_bwd_dq_kernel(const float *__restrict__ acc, uint16_t *__restrict__ dq,
                                 long long n4, float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4 *>(acc)[i];
  reinterpret_cast<uint2 *>(dq)[i] =
      make_uint2(ptx::pack_bf16x2(v.x * scale, v.y * scale), ptx::pack_bf16x2(v.z * scale, v.w * scale));
}

}  // namespace bwd
}  // namespace fa
