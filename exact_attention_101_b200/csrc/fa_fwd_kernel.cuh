// fa_fwd_kernel.cuh -- fused exact-attention forward kernel for B200 (sm_100a).
//
// One persistent CTA per SM walks a static list of work units.  A unit is 256 query
// rows (two 128-row Q tiles) of one (batch, query head); the two tiles share every K/V
// tile that is streamed through shared memory, and their softmax work alternates with
// the tensor core's work on the other tile.  The method is the IO-aware tiled attention
// of the page "FlashAttention (DE)" (sections "Tiling und blockweise Verarbeitung",
// "Online-Softmax-Berechnung", "Zusammenfassen von Operationen in einem CUDA-Kernel"):
// S = Q K^T, the mask, the online softmax and O += P V all happen on chip; only O and
// the per-row log-sum-exp are written.  The warp roles follow the idea of a
// warp-specialised pipeline (page "FlashAttention 4: Praxisleitfaden ...", section "Was
// ist neu in FlashAttention 4?": loading, MMA, softmax, rescaling, epilogue), mapped
// onto sm_100a as follows:
//
//   warps 0-3  softmax + epilogue for Q tile 0 (one thread per query row)
//   warps 4-7  softmax + epilogue for Q tile 1
//   warp  8    tensor-memory allocator and single-thread tcgen05.mma issuer
//   warp  9    single-thread TMA producer
//   warps 10-11 idle (they complete the third warpgroup)
//
// Registers: the kernel is launched with LAUNCH_REGS per thread (384 threads); the
// third warpgroup gives registers back (setmaxnreg.dec to OTHER_REGS) and the two
// softmax warpgroups take them (setmaxnreg.inc to SOFTMAX_REGS), so that a whole score
// row (128 fp32 values) stays in registers.  256*SOFTMAX_REGS + 128*OTHER_REGS equals
// the launch pool 384*LAUNCH_REGS; the host refuses to launch a build whose register
// count would make that sum exceed the pool.
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [  0,128) S0 (fp32 scores of tile 0); P0 (bf16/e4m3 numerators) aliases [64,128)
//   [128,256) S1; P1 aliases [192,256)
//   [256,256+D) O0 accumulator, [256+D, 256+2D) O1 accumulator
//
// Shared memory: Q0, Q1 tiles and a ring of NSLOT K/V tile slots, all in the 128-byte
// swizzled layout that TMA writes and the tensor core reads; plus the mbarriers.
//
// Synchronisation (all mbarriers):
//   q_full / q_empty        Q tiles of a unit loaded / no longer read by an MMA
//   slot_full / slot_empty  ring slot loaded (TMA tx bytes) / released by an MMA commit
//   s_full[x]               S_x of the current key tile is in TMEM
//   p_full[x]               P_x written to TMEM by the 128 softmax threads of tile x
//   o_full[x] / o_empty[x]  O_x final for the unit / read out by the epilogue
//
// Softmax details.  Scores are moved into the base-2 domain with one FFMA,
// x = s * (scale * log2 e), and p = 2^(x - m_used).  m_used is only raised when a key
// tile's row maximum exceeds it by more than RESCALE_THRESHOLD (lazy rescaling, page
// "FlashAttention 4: Praxisleitfaden ...", section "Intelligenteres Online-Softmax-
// Rescaling in FA4"), so p <= 2^RESCALE_THRESHOLD and the accumulator O and the sum l
// are multiplied by 2^(m_old - m_new) only then.  The causal mask is applied only on key
// tiles that cross the diagonal; tiles entirely above it are never loaded.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fa {

// ---------------------------------------------------------------------------- config

constexpr int BM = 128;               // query rows per Q tile (MMA M)
constexpr int BN = 128;               // keys per K/V tile (MMA N of S = Q K^T)
constexpr int UNIT_ROWS = 2 * BM;     // query rows per work unit
constexpr int NUM_THREADS = 384;
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
constexpr int LAUNCH_REGS = 168;    // 65536 / 384, rounded down to a multiple of 8
constexpr int SOFTMAX_REGS = 200;
constexpr int OTHER_REGS = 104;
static_assert(256 * SOFTMAX_REGS + 128 * OTHER_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch pool");
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units: p <= 256

// Error bits written to the device error word when a bounded wait runs out.
constexpr uint32_t ERR_WAIT_SOFTMAX = 1u << 0;
constexpr uint32_t ERR_WAIT_MMA = 1u << 1;
constexpr uint32_t ERR_WAIT_LOAD = 1u << 2;
constexpr uint32_t ERR_WAIT_DRAIN = 1u << 3;

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s per wait
constexpr uint32_t WAIT_MAX_ITERS = 1u << 28;

template <int D, bool FP8>
struct TileCfg {
  static constexpr int ELEM = FP8 ? 1 : 2;           // bytes per element
  static constexpr int ROW_BYTES = D * ELEM;         // bytes per tile row
  static_assert(ROW_BYTES % 128 == 0, "tile rows must be whole 128-byte swizzle rows");
  static constexpr int NBOX = ROW_BYTES / 128;       // 128-byte-wide TMA boxes per row
  static constexpr int BOX_ELEMS = 128 / ELEM;       // elements per box row
  static constexpr int BOX_BYTES = 128 * 128;        // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  static constexpr int NSLOT = TILE_BYTES == 32768 ? 4 : 8;
  static constexpr int MMA_K = FP8 ? 32 : 16;        // K extent of one MMA instruction
  static constexpr int S_KSTEPS = D / MMA_K;         // MMAs per S = Q K^T
  static constexpr int PV_KSTEPS = BN / MMA_K;       // MMAs per O += P V
  static constexpr uint32_t AB_FORMAT = FP8 ? 0u : 1u;  // e4m3 : bf16
  static constexpr uint32_t IDESC_S = ptx::make_idesc(AB_FORMAT, BM, BN, 0);
  static constexpr uint32_t IDESC_O = ptx::make_idesc(AB_FORMAT, BM, D, 1);
  // TMEM column map.
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 128;
  static constexpr uint32_t P_OFF = 64;
  static constexpr uint32_t O_COL0 = 256, O_COL1 = 256 + D;
  static_assert(256 + 2 * D <= (int)TMEM_COLS, "TMEM budget");
  // Shared memory map (offsets from a 1024-aligned base).
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * TILE_BYTES;
  static constexpr int NUM_BARS = 2 * NSLOT + 11;   // + drain barrier
  static constexpr int CTL_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = 1024 + CTL_OFF + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct FwdParams {
  void *o;
  float *lse;
  const float *descale_q;  // fp8 only: [B*Hq]
  const float *descale_k;  // fp8 only: [B*Hkv]
  const float *descale_v;  // fp8 only: [B*Hkv]
  int B, Hq, Hkv, Nq, Nk;
  int group;        // Hq / Hkv
  int num_qb;       // ceil(Nq / UNIT_ROWS)
  int num_units;    // B * Hq * num_qb
  float scale_log2; // softmax scale * log2(e)
};

struct Unit {
  int bh;   // b * Hq + hq
  int bhk;  // b * Hkv + hq / group
  int r0;   // first query row of the unit
  int n0;   // key tiles visited by Q tile 0
  int n1;   // key tiles visited by Q tile 1 (>= n0)
};

// Work list: units of the last query block first (the longest under the causal mask),
// heads in order inside a block so that query heads sharing a K/V head run side by side.
template <bool CAUSAL>
__device__ __forceinline__ Unit decode_unit(const FwdParams &p, int u) {
  const int BH = p.B * p.Hq;
  const int qb = p.num_qb - 1 - u / BH;
  Unit w;
  w.bh = u % BH;
  const int b = w.bh / p.Hq, hq = w.bh % p.Hq;
  w.bhk = b * p.Hkv + hq / p.group;
  w.r0 = qb * UNIT_ROWS;
  const int nkt = (p.Nk + BN - 1) / BN;
  if (CAUSAL) {
    w.n0 = min(p.Nk - 1, w.r0 + BM - 1) / BN + 1;
    w.n1 = min(p.Nk - 1, w.r0 + 2 * BM - 1) / BN + 1;
  } else {
    w.n0 = nkt;
    w.n1 = nkt;
  }
  return w;
}

__device__ unsigned int g_fa_error = 0;

// Bounded wait on an mbarrier phase.  Returns false if another warp of the CTA aborted or
// if this wait ran out (then it raises the CTA abort flag and the device error word).
__device__ __forceinline__ bool wait_phase_slow(uint32_t bar, uint32_t parity,
                                             volatile uint32_t *abort_flag, uint32_t who) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1; it < WAIT_MAX_ITERS; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) break;
    }
  }
  *abort_flag = 1u;
  atomicOr(&g_fa_error, who);
  return false;
}

__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity,
                                           volatile uint32_t *abort_flag, uint32_t who) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_phase_slow(bar, parity, abort_flag, who);
}

// Bounded wait that ignores the abort flag: used to let copies and MMAs already in flight
// land before the CTA frees its tensor memory and exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 0; it < WAIT_MAX_ITERS; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return;
    if ((it & 255u) == 255u && ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) break;
  }
  atomicOr(&g_fa_error, ERR_WAIT_DRAIN);
}

// Barrier addresses in shared memory.
template <int NSLOT>
struct Bars {
  uint32_t base;
  __device__ uint32_t slot_full(int s) const { return base + 8u * s; }
  __device__ uint32_t slot_empty(int s) const { return base + 8u * (NSLOT + s); }
  __device__ uint32_t q_full() const { return base + 8u * (2 * NSLOT + 0); }
  __device__ uint32_t q_empty() const { return base + 8u * (2 * NSLOT + 1); }
  __device__ uint32_t s_full(int x) const { return base + 8u * (2 * NSLOT + 2 + x); }
  __device__ uint32_t p_full(int x) const { return base + 8u * (2 * NSLOT + 4 + x); }
  __device__ uint32_t o_full(int x) const { return base + 8u * (2 * NSLOT + 6 + x); }
  __device__ uint32_t o_empty(int x) const { return base + 8u * (2 * NSLOT + 8 + x); }
};

// ---------------------------------------------------------------------------- producer

template <int D, bool CAUSAL, bool FP8>
__device__ void load_role(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                          const FwdParams &p, uint32_t smem, const Bars<TileCfg<D, FP8>::NSLOT> &bar,
                          volatile uint32_t *abort_flag) {
  using C = TileCfg<D, FP8>;
  ptx::prefetch_tmap(tmQ);
  ptx::prefetch_tmap(tmK);
  ptx::prefetch_tmap(tmV);
  uint32_t issued = 0;    // K/V slot loads issued so far
  uint32_t q_issued = 0;  // Q loads issued so far
  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
    const Unit w = decode_unit<CAUSAL>(p, u);
    if (!wait_phase(bar.q_empty(), (q_issued & 1u) ^ 1u, abort_flag, ERR_WAIT_LOAD)) goto drain;
    ptx::mbar_arrive_expect_tx(bar.q_full(), 2 * C::TILE_BYTES);
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx)
        ptx::tma_load_3d(smem + C::Q_OFF + x * C::TILE_BYTES + bx * C::BOX_BYTES, tmQ,
                         bar.q_full(), bx * C::BOX_ELEMS, w.r0 + x * BM, w.bh);
    ++q_issued;
    for (int j = 0; j < w.n1; ++j) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {  // K_j, then V_j
        const int s = issued % C::NSLOT;
        const uint32_t ph = (issued / C::NSLOT) & 1u;
        if (!wait_phase(bar.slot_empty(s), ph ^ 1u, abort_flag, ERR_WAIT_LOAD)) goto drain;
        ptx::mbar_arrive_expect_tx(bar.slot_full(s), C::TILE_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          ptx::tma_load_3d(smem + C::RING_OFF + s * C::TILE_BYTES + bx * C::BOX_BYTES,
                           t ? tmV : tmK, bar.slot_full(s), bx * C::BOX_ELEMS, j * BN, w.bhk);
        ++issued;
      }
    }
  }
drain:
  // Let every copy this thread started land before the CTA exits (immediate on the normal
  // path, where the consumers have already waited for them).
  for (int s = 0; s < C::NSLOT; ++s) {
    if (issued > (uint32_t)s) {
      const uint32_t last = s + C::NSLOT * ((issued - 1 - s) / C::NSLOT);
      drain_wait(bar.slot_full(s), (last / C::NSLOT) & 1u);
    }
  }
  if (q_issued > 0) drain_wait(bar.q_full(), (q_issued - 1) & 1u);
}

// ---------------------------------------------------------------------------- MMA issuer

template <int D, bool FP8>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_saddr, uint32_t k_saddr) {
  using C = TileCfg<D, FP8>;
#pragma unroll
  for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
    const uint32_t kb = kk * C::MMA_K * C::ELEM;  // byte offset along the head dim
    const uint32_t off = (kb / 128) * C::BOX_BYTES + (kb % 128);
    const uint64_t a = ptx::smem_desc_sw128(q_saddr + off, 16, 1024);
    const uint64_t b = ptx::smem_desc_sw128(k_saddr + off, 16, 1024);
    if (FP8)
      ptx::mma_f8_ss(tmem_s, a, b, C::IDESC_S, kk > 0);
    else
      ptx::mma_bf16_ss(tmem_s, a, b, C::IDESC_S, kk > 0);
  }
}

template <int D, bool FP8>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_saddr,
                                         bool accumulate) {
  using C = TileCfg<D, FP8>;
#pragma unroll
  for (int kk = 0; kk < C::PV_KSTEPS; ++kk) {
    // V is [keys x D] with D contiguous: MN-major B operand.  MMA_K key rows of 128 bytes
    // per step; successive 128-byte D chunks are one TMA box apart.
    const uint64_t b = ptx::smem_desc_sw128(v_saddr + kk * C::MMA_K * 128, C::BOX_BYTES, 1024);
    const uint32_t a = tmem_p + kk * 8;  // 8 TMEM columns hold MMA_K packed P values
    if (FP8)
      ptx::mma_f8_ts(tmem_o, a, b, C::IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
    else
      ptx::mma_bf16_ts(tmem_o, a, b, C::IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool CAUSAL, bool FP8>
__device__ void mma_role(const FwdParams &p, uint32_t smem, uint32_t tmem,
                         const Bars<TileCfg<D, FP8>::NSLOT> &bar, uint32_t drain_bar,
                         volatile uint32_t *abort_flag) {
  using C = TileCfg<D, FP8>;
  const uint32_t q_s[2] = {smem + C::Q_OFF, smem + C::Q_OFF + C::TILE_BYTES};
  const uint32_t t_s[2] = {tmem + C::S_COL0, tmem + C::S_COL1};
  const uint32_t t_p[2] = {tmem + C::S_COL0 + C::P_OFF, tmem + C::S_COL1 + C::P_OFF};
  const uint32_t t_o[2] = {tmem + C::O_COL0, tmem + C::O_COL1};
  uint32_t kv_base = 0;
  uint32_t pph[2] = {0u, 0u};
  uint32_t unit_it = 0;
  auto slot_addr = [&](uint32_t idx) { return smem + C::RING_OFF + (idx % C::NSLOT) * C::TILE_BYTES; };
  auto wait_slot = [&](uint32_t idx) {
    return wait_phase(bar.slot_full(idx % C::NSLOT), (idx / C::NSLOT) & 1u, abort_flag, ERR_WAIT_MMA);
  };
  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x, ++unit_it) {
    const Unit w = decode_unit<CAUSAL>(p, u);
    if (!wait_phase(bar.q_full(), unit_it & 1u, abort_flag, ERR_WAIT_MMA)) break;
    if (!wait_slot(kv_base)) break;
    ptx::tc_fence_after();
    issue_s<D, FP8>(t_s[0], q_s[0], slot_addr(kv_base));
    ptx::mma_commit(bar.s_full(0));
    issue_s<D, FP8>(t_s[1], q_s[1], slot_addr(kv_base));
    ptx::mma_commit(bar.s_full(1));
    ptx::mma_commit(bar.slot_empty(kv_base % C::NSLOT));
    if (w.n1 == 1) ptx::mma_commit(bar.q_empty());
    bool ok = true;
    for (int j = 0; j < w.n1 && ok; ++j) {
      const uint32_t vi = kv_base + 2 * j + 1;  // V_j
      const uint32_t ki = kv_base + 2 * j + 2;  // K_{j+1}
      const bool next = j + 1 < w.n1;
      if (!wait_slot(vi)) { ok = false; break; }
      if (j < w.n0) {
        if (!wait_phase(bar.p_full(0), pph[0], abort_flag, ERR_WAIT_MMA)) { ok = false; break; }
        pph[0] ^= 1u;
        if (j == 0 && !wait_phase(bar.o_empty(0), (unit_it & 1u) ^ 1u, abort_flag, ERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        issue_pv<D, FP8>(t_o[0], t_p[0], slot_addr(vi), j > 0);
        if (j == w.n0 - 1) ptx::mma_commit(bar.o_full(0));
        if (j + 1 < w.n0) {
          if (!wait_slot(ki)) { ok = false; break; }
          ptx::tc_fence_after();
          issue_s<D, FP8>(t_s[0], q_s[0], slot_addr(ki));
          ptx::mma_commit(bar.s_full(0));
        }
      }
      if (!wait_phase(bar.p_full(1), pph[1], abort_flag, ERR_WAIT_MMA)) { ok = false; break; }
      pph[1] ^= 1u;
      if (j == 0 && !wait_phase(bar.o_empty(1), (unit_it & 1u) ^ 1u, abort_flag, ERR_WAIT_MMA)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      issue_pv<D, FP8>(t_o[1], t_p[1], slot_addr(vi), j > 0);
      ptx::mma_commit(bar.slot_empty(vi % C::NSLOT));
      if (j == w.n1 - 1) ptx::mma_commit(bar.o_full(1));
      if (next) {
        if (!wait_slot(ki)) { ok = false; break; }
        ptx::tc_fence_after();
        issue_s<D, FP8>(t_s[1], q_s[1], slot_addr(ki));
        ptx::mma_commit(bar.s_full(1));
        ptx::mma_commit(bar.slot_empty(ki % C::NSLOT));
        if (j + 1 == w.n1 - 1) ptx::mma_commit(bar.q_empty());
      }
    }
    if (!ok) break;
    kv_base += 2 * w.n1;
  }
  // Wait until every MMA issued by this thread has finished before TMEM is freed.
  ptx::mma_commit(drain_bar);
  drain_wait(drain_bar, 0);
}

// ---------------------------------------------------------------------------- softmax

template <int D, bool CAUSAL, bool OUT_F32, bool FP8>
__device__ void softmax_role(const FwdParams &p, uint32_t tmem, const Bars<TileCfg<D, FP8>::NSLOT> &bar,
                             volatile uint32_t *abort_flag) {
  using C = TileCfg<D, FP8>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int x = warp / 4;              // Q tile handled by this warpgroup
  const int wq = warp % 4;             // TMEM lane quarter of this warp
  const int row_in_tile = wq * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t t_s = tmem + lane_base + (x ? C::S_COL1 : C::S_COL0);
  const uint32_t t_p = t_s + C::P_OFF;
  const uint32_t t_o = tmem + lane_base + (x ? C::O_COL1 : C::O_COL0);
  const float NEG_INF = -__int_as_float(0x7f800000);
  uint32_t sph = 0;
  uint32_t unit_it = 0;

  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x, ++unit_it) {
    const Unit w = decode_unit<CAUSAL>(p, u);
    const int nx = x ? w.n1 : w.n0;
    const int row = w.r0 + x * BM + row_in_tile;     // query row of this thread
    const int tile_row0 = w.r0 + x * BM;
    float sl2 = p.scale_log2;
    if (FP8) sl2 *= p.descale_q[w.bh] * p.descale_k[w.bhk];
    // Last admissible key for this row (keys beyond Nk never count).
    const int key_lim = CAUSAL ? min(row, p.Nk - 1) : p.Nk - 1;
    float m_used = NEG_INF;  // running maximum in use, base-2 scaled domain
    float l = 0.f;           // running sum of the numerators as rounded for the P V product
    float l_exact = 0.f;     // running sum of the unrounded numerators (for the LSE)

    for (int j = 0; j < nx; ++j) {
      bool ok = wait_phase(bar.s_full(x), sph, abort_flag, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      sph ^= 1u;
      ptx::tc_fence_after();

      uint32_t sr[8][16];
#pragma unroll
      for (int c = 0; c < 8; ++c) ptx::tmem_ld16(t_s + c * 16, sr[c]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 8; ++c) ptx::reg_fence16(sr[c]);

      const int kv0 = j * BN;
      const bool need_mask = (CAUSAL && kv0 + BN - 1 > tile_row0) || (kv0 + BN > p.Nk);
      if (need_mask) {
        const int lim = key_lim - kv0;  // column c is admissible iff c <= lim
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c * 16 + e > lim) sr[c][e] = __float_as_uint(NEG_INF);
      }
      // Row maximum (4 independent chains).
      float mx[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(sr[c][e]));
      const float xmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;

      // Lazy rescale: move m_used only when the new maximum is far above it.
      const bool resc = xmax > m_used + RESCALE_THRESHOLD;
      const float alpha = resc ? ptx::ex2(m_used - xmax) : 1.f;  // 0 on the first tile
      if (__any_sync(0xffffffffu, resc && j > 0)) {
        // O_x is quiescent here: the commit that signalled S_x(j) covers the MMA that
        // accumulated P_x(j-1) V(j-1), and P_x(j) V(j) waits for p_full below.
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o[16];
          ptx::tmem_ld16(t_o + c * 16, o);
          ptx::tmem_wait_ld();
          ptx::reg_fence16(o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          ptx::tmem_st16(t_o + c * 16, o);
        }
        ptx::tmem_wait_st();
      }
      if (resc) {
        l *= alpha;
        l_exact *= alpha;
        m_used = xmax;
      }
      const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used;

      // Numerators p = 2^(s*sl2 - m_used), packed for the P V product.
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      float le[4] = {0.f, 0.f, 0.f, 0.f};
      if (!FP8) {
        uint32_t pk[4][16];
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[c][e]), sl2, neg_m));
            const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m));
            const uint32_t pp = ptx::pack_bf16x2(p0, p1);
            const int col = c * 8 + e / 2;
            pk[col / 16][col % 16] = pp;
            // l sums the same rounded values the tensor core multiplies with V, so that O
            // stays a convex combination of value rows; l_exact keeps the LSE accurate.
            ls[(e / 2) & 3] += __uint_as_float(pp << 16) + __uint_as_float(pp & 0xffff0000u);
            le[(e / 2) & 3] += p0 + p1;
          }
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_st16(t_p + c * 16, pk[c]);
      } else {
        uint32_t pk[2][16];
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[c][e]), sl2, neg_m));
            const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m));
            const float p2 = ptx::ex2(fmaf(__uint_as_float(sr[c][e + 2]), sl2, neg_m));
            const float p3 = ptx::ex2(fmaf(__uint_as_float(sr[c][e + 3]), sl2, neg_m));
            const int col = c * 4 + e / 4;
            pk[col / 16][col % 16] = ptx::pack_e4m3x4(p0, p1, p2, p3);
            le[(e / 4) & 3] += (p0 + p1) + (p2 + p3);
          }
#pragma unroll
        for (int c = 0; c < 2; ++c) ptx::tmem_st16(t_p + c * 16, pk[c]);
      }
      l_exact += (le[0] + le[1]) + (le[2] + le[3]);
      if (FP8)
        l = l_exact;
      else
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar.p_full(x));
    }

    // Epilogue: O = O_acc / l (times the V descale for fp8),
    // LSE = ln 2 * (m_used + log2 l_exact).
    {
      bool ok = wait_phase(bar.o_full(x), unit_it & 1u, abort_flag, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      ptx::tc_fence_after();
      float inv = 1.f / l;
      if (FP8) inv *= p.descale_v[w.bhk];
      const bool valid = row < p.Nq;
      const size_t orow = static_cast<size_t>(w.bh) * p.Nq + (valid ? row : 0);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[16], b[16];
        ptx::tmem_ld16(t_o + c * 32, a);
        ptx::tmem_ld16(t_o + c * 32 + 16, b);
        ptx::tmem_wait_ld();
        ptx::reg_fence16(a);
        ptx::reg_fence16(b);
        if (valid) {
          if (OUT_F32) {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow * D + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_float4(__uint_as_float(a[4 * v]) * inv, __uint_as_float(a[4 * v + 1]) * inv,
                                   __uint_as_float(a[4 * v + 2]) * inv, __uint_as_float(a[4 * v + 3]) * inv);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[4 + v] = make_float4(__uint_as_float(b[4 * v]) * inv, __uint_as_float(b[4 * v + 1]) * inv,
                                       __uint_as_float(b[4 * v + 2]) * inv, __uint_as_float(b[4 * v + 3]) * inv);
          } else {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow * D + c * 32);
            uint32_t h[16];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              h[e] = ptx::pack_bf16x2(__uint_as_float(a[2 * e]) * inv, __uint_as_float(a[2 * e + 1]) * inv);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              h[8 + e] = ptx::pack_bf16x2(__uint_as_float(b[2 * e]) * inv, __uint_as_float(b[2 * e + 1]) * inv);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
          }
        }
      }
      if (valid) p.lse[orow] = (m_used + log2f(l_exact)) * 0.69314718055994530942f;
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar.o_empty(x));
    }
  }
}

// ---------------------------------------------------------------------------- kernel

template <int D, bool CAUSAL, bool OUT_F32, bool FP8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = TileCfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t smem = (raw + 1023u) & ~1023u;  // 1024-aligned for 128-byte swizzle
  uint8_t *smem_gen = smem_raw + (smem - raw);
  const Bars<C::NSLOT> bar{smem + C::BAR_OFF};
  const uint32_t drain_bar = smem + C::BAR_OFF + 8u * (C::NUM_BARS - 1);
  uint32_t *ctl = reinterpret_cast<uint32_t *>(smem_gen + C::CTL_OFF);
  volatile uint32_t *tmem_slot = ctl;
  volatile uint32_t *abort_flag = ctl + 1;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      ptx::mbar_init(bar.slot_full(s), 1);
      ptx::mbar_init(bar.slot_empty(s), 1);
    }
    ptx::mbar_init(bar.q_full(), 1);
    ptx::mbar_init(bar.q_empty(), 1);
    for (int x = 0; x < 2; ++x) {
      ptx::mbar_init(bar.s_full(x), 1);
      ptx::mbar_init(bar.p_full(x), BM);
      ptx::mbar_init(bar.o_full(x), 1);
      ptx::mbar_init(bar.o_empty(x), BM);
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    ptx::tmem_alloc(ptx::smem_addr(ctl), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8)
    ptx::setmaxnreg_inc<SOFTMAX_REGS>();
  else
    ptx::setmaxnreg_dec<OTHER_REGS>();

  if (warp < 8) {
    softmax_role<D, CAUSAL, OUT_F32, FP8>(p, tmem, bar, abort_flag);
  } else if (warp == MMA_WARP) {
    if (lane == 0) mma_role<D, CAUSAL, FP8>(p, smem, tmem, bar, drain_bar, abort_flag);
    __syncwarp();
  } else if (warp == TMA_WARP) {
    if (lane == 0) load_role<D, CAUSAL, FP8>(&tmQ, &tmK, &tmV, p, smem, bar, abort_flag);
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fa
