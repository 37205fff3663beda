// fa_fwd_pair.cuh -- the bf16 attention forward on CTA pairs, head dims 128 and 256
// (sm_100a).
//
// The library runs it at head dim 128 without the causal mask (causal work there goes to
// the one-CTA kernel, which measured faster; the pair's causal instance at 128 is built with
// FA_PAIR_CAUSAL only) and at head dim 256 with or without it.  The text below describes
// D = 128; PCfg gives what changes at D = 256 (four Q boxes and one Q buffer, 32 KB ring
// slots, a V half of 128 dimensions, O of 256 columns and P over the first columns of S).
//
// Same method as fa_fwd_kernel.cuh (the IO-aware tiled attention of the page "FlashAttention
// (DE)", sections "Tiling und blockweise Verarbeitung", "Online-Softmax-Berechnung" and
// "Zusammenfassen von Operationen in einem CUDA-Kernel"; the warp roles of the page
// "FlashAttention 4: Praxisleitfaden ...", section "Was ist neu in FlashAttention 4?"), laid
// out for the tensor core's two-SM products.
//
// Why pairs.  A one-SM S = Q K^T product with M = 128 reads A (Q) and B (K) from shared
// memory: at N = 64 keys that is 6 KB per 32 tensor-core cycles, above the 128 bytes per
// cycle that shared memory delivers, so the one-SM kernel is bound by shared-memory
// bandwidth (about 160 KB per 64-key step against 1024 tensor cycles).  A pair of CTAs on
// two SMs issues tcgen05 products with M = 256 (.cta_group::2): each SM holds 128 rows of A
// and half of B's N columns, and computes its own 128 rows of D.  With 128-key blocks a
// K-step reads 4 KB of Q and 2 KB of K per SM for 64 cycles; V is split the same way, and
// each CTA loads only its halves of K and V.  Per 128-key block an SM moves about 80 KB
// through shared memory for 1024 tensor cycles.
//
// Geometry.  A cluster of two CTAs (ranks 0 and 1) processes a unit of 256 query rows of
// one (batch, query head), rows [128 r, 128 r + 128) in CTA r (its 128 tensor-memory
// lanes).  Keys come in blocks of BN = 128; CTA r holds keys [64 r, 64 r + 64) of every K
// block (all 128 dimensions) and dimensions [64 r, 64 r + 64) of every V block (all 128
// keys).  Per CTA:
//
//   warps 0-3   softmax of the even key blocks (key stream 0), and the epilogue of O's
//               dimensions 0-63 (thread = query row = TMEM lane)
//   warps 4-7   the odd key blocks (stream 1), and dimensions 64-127
//   warp  8     tensor-memory allocator; in CTA 0 the MMA issuer
//   warp  9     TMA producer (lane 0); in CTA 0 also the claimer of work units
//   warps 10-11 idle (complete the third warpgroup)
//
// Two key streams.  At head dim 128 the exponentials of a block take the SFU as long as the
// tensor core takes for the block's two products (16 exponentials and 16 x 512 MMA FLOPs
// per SM per cycle), and one warp's softmax of a 128-key block also waits on tensor-memory
// loads and stores.  So the two softmax warpgroups take turns: warpgroup s handles the
// blocks j with j mod 2 == s, full 128-key rows, while the other loads and exponentiates its
// own block.  Both use one running maximum: block j's maximum in use is handed to block
// j+1 through shared memory right after block j's row maximum is known (lazy rescaling: it
// only moves when the block maximum exceeds it by more than RESCALE_THRESHOLD), so the
// numerators of every block are relative to the maximum O holds.  Each warpgroup keeps its
// own part of the row sum, brought to the final maximum and added in the epilogue.
//
// Tensor memory (512 columns, allocated for the pair): score buffers S(b) at b * 128 (128
// fp32 columns), the accumulator O at 256, numerator buffers P(b) at 384 + b * 64 (bf16
// pairs).  P does not overwrite S, so S(j+2) is computed into S(j mod 2) as soon as the
// softmax has read S(j), while block j's numerators are still being formed: the softmax
// then finds its next scores ready.
//
// MMA order inside a unit (one warp of CTA 0): S(0), S(1), then for every block j: S(j+2)
// once S(j) has been read, then P(j) V_j into O once P(j) is written.  O is rescaled (by
// the softmax of block j, rarely) only after P(j-1) V has completed (pv_done) and before
// P(j) V is issued.
//
// Synchronisation.  Barriers sit at the same offsets in both CTAs.  Those the MMA warp waits
// on live in CTA 0 (slot_full, q_full, s_free, p_full, o_empty, unit_empty): both CTAs'
// copies signal CTA 0's slot_full/q_full (.cta_group::2 copies), and CTA 1's softmax warps
// arrive on CTA 0's s_free/p_full/o_empty remotely.  Those the producers and softmax warps
// wait on are signalled in both CTAs at once by the MMA commits (slot_empty, q_empty,
// s_full, pv_done, o_full).  CTA 0's producer claims units and writes each into both CTAs'
// unit rings.  The maximum handoff and the epilogue's sum exchange stay inside a CTA.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {
namespace pair {

constexpr int BM = 128;                     // query rows of a unit held by one CTA
constexpr int BN = 128;                     // keys per block (N of S over the pair)
constexpr int UNIT_ROWS = 2 * BM;           // query rows per unit (MMA M)
constexpr int NUM_THREADS = 384;
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 208;
constexpr int OTHER_REGS = (NUM_THREADS * LAUNCH_REGS - 256 * SOFTMAX_REGS) / 128 / 8 * 8;
static_assert(OTHER_REGS >= 64, "register split leaves too few for the MMA/TMA warps");
static_assert(256 * SOFTMAX_REGS + 128 * OTHER_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch pool");
#ifndef FA_PAIR_POLY_PAIRS
#define FA_PAIR_POLY_PAIRS 0
#endif
// Column pairs (of every 8) whose exponentials use the FMA-pipe polynomial instead of the
// SFU, on blocks without masked entries.
constexpr int POLY_PAIRS = FA_PAIR_POLY_PAIRS;
static_assert(POLY_PAIRS >= 0 && POLY_PAIRS <= 8, "pairs per 16-column chunk");
constexpr uint32_t TMEM_COLS = 512;
constexpr int Q_BOX_BYTES = BM * 128;       // 128 rows x 128 bytes (64 dims)
constexpr int K_BOX_BYTES = 64 * 128;       // 64 keys x 128 bytes (64 dims)
constexpr int V_BOX_BYTES = BN * 128;       // 128 keys x 128 bytes (64 dims)
constexpr int PV_KSTEPS = BN / 16;
constexpr uint32_t IDESC_S = ptx::make_idesc(1u, 256, BN, 0);
constexpr int UNIT_RING_P = 4;
// consumers of a published unit: CTA 0's MMA warp and eight softmax warps, CTA 1's eight
// softmax warps and its producer
constexpr uint32_t UNIT_CONSUMERS = 1 + 8 + 8 + 1;
constexpr uint32_t SOFTMAX_WARPS_PAIR = 16;  // softmax warps of both CTAs (o_empty)
constexpr uint32_t STREAM_WARPS_PAIR = 8;    // one stream's softmax warps, both CTAs
constexpr uint16_t BOTH = 0x3;              // CTA mask of the pair
// the per-row maximum handed between the streams [2 streams][128 rows] (and the exact
// running maximum, for the rescale statistics) and the epilogue's sum exchange [2
// streams][128 rows], fp32
constexpr int XCH_BYTES = 3 * 2 * BM * 4;
constexpr int STAGE_WARP_BYTES = 32 * 64;   // epilogue staging: 32 rows x 64 bytes per warp

// Layout for head dimension D (128 or 256).
//   Q: this CTA's 128 rows in D/64 boxes of 64 dims; two buffers (unit parity) at D = 128,
//      one at D = 256 (the next unit's Q then loads after the unit's last S).
//   Ring slot: a K half (64 keys x D dims, D/64 boxes) or a V half (128 keys x D/2 dims,
//      D/128 boxes of 64 dims); 128 KB of slots.
//   Tensor memory: S(b) at 128 b (128 fp32 columns), O at 256 (D columns), and the bf16
//      numerators P(b): at D = 128 in their own columns (384 + 64 b), so that S(j+2) can be
//      computed while block j's numerators are still being formed; at D = 256 O takes the
//      last 256 columns, so P(b) goes over the first 64 columns of S(b), and S(j+2) waits
//      until P(j) V has been issued (products of one thread run in issue order).
template <int D>
struct PCfg {
  static_assert(D == 128 || D == 256, "head dims of the pair kernel");
  static constexpr int NQBOX = D / 64;
  static constexpr int Q_TILE_BYTES = NQBOX * Q_BOX_BYTES;
  static constexpr int NQBUF = D == 128 ? 2 : 1;
  static constexpr int NKBOX = D / 64;
  static constexpr int NVBOX = D / 128;
  static constexpr int SLOT_BYTES = NKBOX * K_BOX_BYTES;
  static_assert(NVBOX * V_BOX_BYTES == SLOT_BYTES, "K and V halves fill one slot");
  static constexpr int NSLOT = 131072 / SLOT_BYTES;
  static constexpr int S_KSTEPS = D / 16;
  static constexpr uint32_t IDESC_O = ptx::make_idesc(1u, 256, D, 1);
  static constexpr bool ALIAS_P = D == 256;
  static constexpr uint32_t O_COL0 = 256;
  __host__ __device__ static constexpr uint32_t p_col(int b) {
    return ALIAS_P ? 128u * b : 384u + 64u * b;
  }
  // S(k) may be issued once P(k - 1 - S_LEAD) V has been issued: at D = 128 that keeps every
  // pv_done barrier at most one phase ahead of the softmax's parity waits; at D = 256 it also
  // keeps S(k) behind the P V that reads P(k-2) from the same columns
  static constexpr int S_LEAD = ALIAS_P ? 1 : 2;
  static_assert(O_COL0 + D <= TMEM_COLS, "TMEM budget");
  // shared memory: the Q buffers, the K/V ring, the exchange, the epilogue staging, the
  // mbarriers and the control words
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NQBUF * Q_TILE_BYTES;
  static constexpr int XCH_OFF = RING_OFF + NSLOT * SLOT_BYTES;
  static constexpr int STAGE_OFF = XCH_OFF + XCH_BYTES;
  static constexpr int BAR_OFF = STAGE_OFF + 8 * STAGE_WARP_BYTES;
  static constexpr int NUM_BARS = 2 * NSLOT + 27 + 2 * UNIT_RING_P;
  static constexpr int CTL_OFF = BAR_OFF + NUM_BARS * 8;
  // control words: TMEM base, abort flag, 2 spare, then the unit ring
  static constexpr int SMEM_BYTES = 1024 + CTL_OFF + 16 + 4 * UNIT_RING_P;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int NSLOT>
struct PBars {
  uint32_t base;
  __device__ uint32_t slot_full(int s) const { return base + 8u * s; }
  __device__ uint32_t slot_empty(int s) const { return base + 8u * (NSLOT + s); }
  __device__ uint32_t at(int i) const { return base + 8u * (2 * NSLOT + i); }
  __device__ uint32_t q_full(int q) const { return at(q); }
  __device__ uint32_t q_empty(int q) const { return at(2 + q); }
  __device__ uint32_t s_full(int b) const { return at(4 + b); }    // S(b) computed
  __device__ uint32_t s_free(int b) const { return at(6 + b); }    // S(b) read by the softmax
  __device__ uint32_t p_full(int b) const { return at(8 + b); }    // P(b) written
  __device__ uint32_t pv_done(int b) const { return at(10 + b); }  // P(b) V completed
  __device__ uint32_t o_full() const { return at(12); }
  __device__ uint32_t o_empty() const { return at(13); }
  __device__ uint32_t drain() const { return at(14); }
  // epilogue sum exchange of warp pair (wq, wq + 4), wq = 0..3
  __device__ uint32_t xchg(int wq) const { return at(15 + wq); }
  // maximum published by stream s for the rows of lane quarter wq
  __device__ uint32_t hand(int s, int wq) const { return at(19 + 4 * s + wq); }
  __device__ uint32_t unit_full(int s) const { return at(27 + s); }
  __device__ uint32_t unit_empty(int s) const { return at(27 + UNIT_RING_P + s); }
};

// The CTA's abort flag and its address in the peer CTA: a wait that gives up raises both,
// so that the peer stops waiting for work this CTA will not do.
struct Abort {
  volatile uint32_t *flag;
  uint32_t peer;  // shared::cluster address of the peer's flag
};

template <bool CLUSTER>
__device__ __forceinline__ bool pwait_slow(uint32_t bar, uint32_t parity, const Abort &ab,
                                           uint32_t who) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1; it < WAIT_MAX_ITERS; ++it) {
    if (CLUSTER ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity))
      return true;
    if ((it & 255u) == 0) {
      if (*ab.flag) return false;
      if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) break;
    }
  }
  *ab.flag = 1u;
  ptx::st_cluster_u32(ab.peer, 1u);
  atomicOr(&g_fa_error, who);
  return false;
}

// Bounded wait on a phase of one of this CTA's mbarriers.  The per-block handshakes use
// the default (CTA-scope acquire) semantics: what they hand over is tensor memory or MMA
// operands, ordered by tcgen05 fences and the async proxy.  The unit ring, whose value is
// an ordinary shared-memory word written by the other CTA, waits with cluster-scope
// acquire (CLUSTER).
template <bool CLUSTER = false>
__device__ __forceinline__ bool pwait(uint32_t bar, uint32_t parity, const Abort &ab,
                                      uint32_t who) {
  if (CLUSTER ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity))
    return true;
  return pwait_slow<CLUSTER>(bar, parity, ab, who);
}

// Key blocks that query rows up to `last_row` visit (at least one; see key_tiles).
template <bool CAUSAL>
__device__ __forceinline__ int key_blocks(int last_row, int len_k, int off) {
  const int last_key = CAUSAL ? min(len_k - 1, last_row + off) : len_k - 1;
  return last_key < 0 ? 1 : last_key / BN + 1;
}

struct PUnit {
  int bh;    // b * Hq + hq
  int bhk;   // b * Hkv + hq / group
  int r0;    // first query row of the unit
  int off;   // causal diagonal: query i sees keys j <= i + off
  int n;     // key blocks the unit visits
};

// Work list as in decode_unit: head by head without the mask; under the causal mask groups
// of CAUSAL_HEAD_GROUP heads, longest units first.
template <bool CAUSAL>
__device__ __forceinline__ PUnit pair_decode(const FwdParams &p, int u) {
  constexpr int HG = CAUSAL ? CAUSAL_HEAD_GROUP : 1;
  const int BH = p.num_units / p.num_qb;
  const int g = u / (HG * p.num_qb);
  const int r = u - g * HG * p.num_qb;
  const int heads = min(HG, BH - g * HG);
  const int qb = p.num_qb - 1 - r / heads;
  PUnit w;
  w.bh = g * HG + r % heads;
  const int b = w.bh / p.Hq, hq = w.bh % p.Hq;
  w.bhk = b * p.Hkv + hq / p.group;
  w.r0 = qb * UNIT_ROWS;
  w.off = p.Nk - p.Nq;
  w.n = key_blocks<CAUSAL>(w.r0 + UNIT_ROWS - 1, p.Nk, w.off);
  return w;
}

// ---------------------------------------------------------------------------- producer

// Lane 0 of warp 9 in both CTAs.  CTA 0 claims units (its first is its cluster index, then
// one atomic per unit) and publishes each in both CTAs' rings; CTA 1 takes them from its
// ring.  Each CTA copies its own 128 rows of Q (into the buffer of the unit's parity) and
// its halves of every K and V block; all copies complete on CTA 0's barriers, which CTA 0
// arms with the bytes of both.
template <int D, bool CAUSAL>
__device__ void pair_load_role(const CUtensorMap *tmQ, const CUtensorMap *tmK,
                               const CUtensorMap *tmV, const FwdParams &p, uint32_t smem,
                               const PBars<PCfg<D>::NSLOT> &bar, volatile uint32_t *ring,
                               const Abort &ab, uint32_t rank) {
  using C = PCfg<D>;
  constexpr int NSLOT = C::NSLOT;
  ptx::prefetch_tmap(tmQ);
  ptx::prefetch_tmap(tmK);
  ptx::prefetch_tmap(tmV);
  const uint32_t num_units = static_cast<uint32_t>(p.num_units);
  uint32_t issued = 0, q_issued = 0, units = 0;
  uint32_t u = ptx::cluster_id_x();
  for (;;) {
    const int s = units % UNIT_RING_P;
    const uint32_t ph = (units / UNIT_RING_P) & 1u;
    if (rank == 0) {  // publish u (or, past the last unit, the end of the list)
      if (!pwait<true>(bar.unit_empty(s), ph ^ 1u, ab, ERR_WAIT_LOAD)) goto drain;
      ring[s] = u;
      ptx::st_cluster_u32(ptx::mapa(ptx::smem_addr(const_cast<uint32_t *>(ring + s)), 1), u);
      ptx::mbar_arrive(bar.unit_full(s));
      ptx::mbar_arrive_cluster(ptx::mapa(bar.unit_full(s), 1));
    } else {
      if (!pwait<true>(bar.unit_full(s), ph, ab, ERR_WAIT_LOAD)) goto drain;
      u = ring[s];
      ptx::mbar_arrive_cluster(ptx::mapa(bar.unit_empty(s), 0));
    }
    ++units;
    if (u >= num_units) break;
    {
      const PUnit w = pair_decode<CAUSAL>(p, static_cast<int>(u));
      const int qb = q_issued % C::NQBUF;
      if (!pwait(bar.q_empty(qb), ((q_issued / C::NQBUF) & 1u) ^ 1u, ab, ERR_WAIT_LOAD))
        goto drain;
      if (rank == 0) ptx::mbar_arrive_expect_tx(bar.q_full(qb), 2 * C::Q_TILE_BYTES);
      const uint32_t qf = ptx::mapa(bar.q_full(qb), 0);
#pragma unroll
      for (int bx = 0; bx < C::NQBOX; ++bx)
        ptx::tma_load_3d_pair(smem + C::Q_OFF + qb * C::Q_TILE_BYTES + bx * Q_BOX_BYTES, tmQ,
                              qf, bx * 64, w.r0 + static_cast<int>(rank) * BM, w.bh);
      ++q_issued;
      // K and V halves in the order the MMA warp first needs them: K_0, K_1, then per block
      // j K_(j+2) (its scores are computed early) and V_j
      auto load_k = [&](int j) -> bool {
        const int sl = issued % NSLOT;
        if (!pwait(bar.slot_empty(sl), ((issued / NSLOT) & 1u) ^ 1u, ab, ERR_WAIT_LOAD))
          return false;
        if (rank == 0) ptx::mbar_arrive_expect_tx(bar.slot_full(sl), 2 * C::SLOT_BYTES);
        const uint32_t sf = ptx::mapa(bar.slot_full(sl), 0);
        // keys j*BN + 64 rank .. + 63, all dimensions (D/64 boxes of 64 dimensions)
#pragma unroll
        for (int bx = 0; bx < C::NKBOX; ++bx)
          ptx::tma_load_3d_pair(smem + C::RING_OFF + sl * C::SLOT_BYTES + bx * K_BOX_BYTES, tmK,
                                sf, bx * 64, j * BN + static_cast<int>(rank) * 64, w.bhk);
        ++issued;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int sl = issued % NSLOT;
        if (!pwait(bar.slot_empty(sl), ((issued / NSLOT) & 1u) ^ 1u, ab, ERR_WAIT_LOAD))
          return false;
        if (rank == 0) ptx::mbar_arrive_expect_tx(bar.slot_full(sl), 2 * C::SLOT_BYTES);
        const uint32_t sf = ptx::mapa(bar.slot_full(sl), 0);
        // keys j*BN .. + 127, dimensions (D/2) rank .. + D/2 - 1 (D/128 boxes of 64 dimensions)
#pragma unroll
        for (int bx = 0; bx < C::NVBOX; ++bx)
          ptx::tma_load_3d_pair(smem + C::RING_OFF + sl * C::SLOT_BYTES + bx * V_BOX_BYTES, tmV,
                                sf, static_cast<int>(rank) * (D / 2) + bx * 64, j * BN, w.bhk);
        ++issued;
        return true;
      };
      if (!load_k(0)) goto drain;
      if (w.n > 1 && !load_k(1)) goto drain;
      for (int j = 0; j < w.n; ++j) {
        if (C::ALIAS_P) {
          if (!load_v(j)) goto drain;
          if (j + 2 < w.n && !load_k(j + 2)) goto drain;
        } else {
          if (j + 2 < w.n && !load_k(j + 2)) goto drain;
          if (!load_v(j)) goto drain;
        }
      }
    }
    if (rank == 0) u = ptx::num_clusters_x() + atomicAdd(p.sched, 1u);
  }
drain:
  if (rank == 0) {
    // every phase this CTA armed completes once both CTAs' copies have landed
    for (int s = 0; s < NSLOT; ++s) {
      if (issued > static_cast<uint32_t>(s)) {
        const uint32_t last = s + NSLOT * ((issued - 1 - s) / NSLOT);
        drain_wait(bar.slot_full(s), (last / NSLOT) & 1u);
      }
    }
    for (uint32_t qb = 0; qb < C::NQBUF; ++qb) {
      if (q_issued > qb) {
        const uint32_t last = qb + C::NQBUF * ((q_issued - 1 - qb) / C::NQBUF);
        drain_wait(bar.q_full(qb), (last / C::NQBUF) & 1u);
      }
    }
  } else if (*ab.flag) {
    // After an abort CTA 1 cannot see CTA 0's barriers: give copies it issued for phases
    // CTA 0 never armed time to land before the CTAs leave (bounded, 200 us).
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 0; it < WAIT_MAX_ITERS && ptx::globaltimer_ns() - t0 < 200000ull; ++it) {
    }
  }
}

// ---------------------------------------------------------------------------- MMA issuer

template <int D>
__device__ __forceinline__ void pair_issue_s(uint32_t tmem_s, uint64_t q_desc, uint64_t k_desc) {
#pragma unroll
  for (int kk = 0; kk < PCfg<D>::S_KSTEPS; ++kk) {
    const uint32_t kb = kk * 32;  // bytes along the head dimension
    const uint32_t qoff = ((kb / 128) * Q_BOX_BYTES + (kb % 128)) >> 4;
    const uint32_t koff = ((kb / 128) * K_BOX_BYTES + (kb % 128)) >> 4;
    ptx::mma2_bf16_ss_elect(tmem_s, q_desc + qoff, k_desc + koff, IDESC_S, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void pair_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t v_desc,
                                              uint32_t accumulate) {
  // V half is [128 keys x D/2 dims], dims contiguous: an MN-major B operand of D/128 swizzle
  // atoms (128-byte dimension chunks, one box apart: the LBO of v_desc) across N; 16 key rows
  // of 128 bytes per K-step.
#pragma unroll
  for (int kk = 0; kk < PV_KSTEPS; ++kk) {
    const uint32_t off = (kk * 16 * 128) >> 4;
    ptx::mma2_bf16_ts_elect(tmem_o, tmem_p + kk * 8, v_desc + off, PCfg<D>::IDESC_O,
                            kk > 0 ? 1u : accumulate);
  }
}

// Ring position, inside a unit of n key blocks, of K_k and V_j in the producer's order, the
// order in which the MMA warp first needs them: K_0, K_1, then per block j K_(j+2) (while
// j + 2 < n) and V_j -- or, where S(j+2) follows P(j) V (P over S, D = 256), V_j and K_(j+2).
template <int D>
__device__ __forceinline__ uint32_t k_pos(int k) {
  return k < 2 ? k : (PCfg<D>::ALIAS_P ? 2 * k - 1 : 2 * k - 2);
}
template <int D>
__device__ __forceinline__ uint32_t v_pos(int j, int n) {
  return (n > 1 ? 2 : 1) + j + min(PCfg<D>::ALIAS_P ? j : j + 1, max(n - 2, 0));
}

// Warp 8 of CTA 0.  Every commit that frees a resource or signals a result arrives on the
// barrier in both CTAs.  Inside a unit it issues, in a loop of non-blocking probes,
// whichever product can go next: S(k) once its buffer has been read (s_free of block k-2),
// K_k has landed and P(k-3) V has been issued, or P(j) V_j once the numerators P(j) are
// written -- so scores for the next blocks never queue behind a product that waits for the
// softmax.
template <int D, bool CAUSAL>
__device__ void pair_mma_role(const FwdParams &p, uint32_t smem, uint32_t tmem,
                              const PBars<PCfg<D>::NSLOT> &bar, volatile uint32_t *ring,
                              const Abort &ab) {
  using C = PCfg<D>;
  constexpr int NSLOT = C::NSLOT;
  const uint64_t q_d0 = ptx::smem_desc_sw128(smem + C::Q_OFF, 16, 1024);
  const uint64_t k_d0 = ptx::smem_desc_sw128(smem + C::RING_OFF, 16, 1024);
  const uint64_t v_d0 = ptx::smem_desc_sw128(smem + C::RING_OFF, V_BOX_BYTES, 1024);
  constexpr uint32_t SLOT_STEP = C::SLOT_BYTES >> 4;
  constexpr uint32_t QBUF_STEP = C::Q_TILE_BYTES >> 4;
  uint32_t kv_base = 0, unit_it = 0, taken = 0;
  uint32_t pph = 0;           // phase bits of p_full(b), bit b
  uint32_t sfph = 0;          // phase bits of s_free(b), bit b
  uint32_t s_issued = 0;      // bit b: an S product has been issued into buffer b
  bool ok = true;
  auto wait = [&](uint32_t b, uint32_t parity) {
    const bool r = pwait(b, parity, ab, ERR_WAIT_MMA);
    return __all_sync(0xffffffffu, r);
  };
  // warp-uniform non-blocking probe
  auto ready = [&](uint32_t b, uint32_t parity) {
    return __all_sync(0xffffffffu, ptx::mbar_test_wait(b, parity));
  };
  auto slot_ready = [&](uint32_t idx) {
    return ready(bar.slot_full(idx % NSLOT), (idx / NSLOT) & 1u);
  };
  while (ok) {
    const int s = taken % UNIT_RING_P;
    if (!__all_sync(0xffffffffu, pwait<true>(bar.unit_full(s), (taken / UNIT_RING_P) & 1u, ab,
                                             ERR_WAIT_MMA)))
      break;
    const uint32_t u = ring[s];
    __syncwarp();
    ptx::mbar_arrive_elect(bar.unit_empty(s));
    ++taken;
    if (u >= static_cast<uint32_t>(p.num_units)) break;
    const PUnit w = pair_decode<CAUSAL>(p, static_cast<int>(u));
    const int n = w.n;
    const int qb = unit_it % C::NQBUF;
    const uint64_t q_d = q_d0 + qb * QBUF_STEP;
    if (!wait(bar.q_full(qb), (unit_it / C::NQBUF) & 1u)) break;
    int next_s = 0, next_pv = 0;
    uint64_t t_idle = 0;  // start of the current run of probes without progress
    uint32_t spins = 0;
    while (next_pv < n) {
      bool progressed = false;
      // S(k) only after P(k-1-S_LEAD) V has been issued: products of one thread complete in
      // order, so when the softmax sees S(k), every pv_done barrier has at most one pending
      // phase (P(k-1) V or P(k-2) V), which its parity waits rely on; where P shares S's
      // columns (S_LEAD 1), S(k) also follows the P(k-2) V that reads them
      if (next_s < n && next_s <= next_pv + C::S_LEAD) {
        const int k = next_s, b = k & 1;
        const bool buf_free = !((s_issued >> b) & 1u) || ready(bar.s_free(b), (sfph >> b) & 1u);
        const uint32_t ki = kv_base + k_pos<D>(k);
        if (buf_free && slot_ready(ki)) {
          if ((s_issued >> b) & 1u) sfph ^= 1u << b;
          ptx::tc_fence_after();
          pair_issue_s<D>(tmem + b * BN, q_d, k_d0 + (ki % NSLOT) * SLOT_STEP);
          ptx::mma2_commit_mc_elect(bar.s_full(b), BOTH);
          ptx::mma2_commit_mc_elect(bar.slot_empty(ki % NSLOT), BOTH);
          if (k == n - 1) ptx::mma2_commit_mc_elect(bar.q_empty(qb), BOTH);
          s_issued |= 1u << b;
          ++next_s;
          progressed = true;
        }
      }
      if (next_pv < next_s) {
        const int j = next_pv, b = j & 1;
        const uint32_t vi = kv_base + v_pos<D>(j, n);
        // the previous unit's epilogue has read O before P(0) V overwrites it
        if (ready(bar.p_full(b), (pph >> b) & 1u) && slot_ready(vi) &&
            (j > 0 || ready(bar.o_empty(), (unit_it & 1u) ^ 1u))) {
          pph ^= 1u << b;
          ptx::tc_fence_after();
          pair_issue_pv<D>(tmem + C::O_COL0, tmem + C::p_col(b), v_d0 + (vi % NSLOT) * SLOT_STEP,
                           j > 0 ? 1u : 0u);
          ptx::mma2_commit_mc_elect(bar.pv_done(b), BOTH);
          ptx::mma2_commit_mc_elect(bar.slot_empty(vi % NSLOT), BOTH);
          if (j == n - 1) ptx::mma2_commit_mc_elect(bar.o_full(), BOTH);
          ++next_pv;
          progressed = true;
        }
      }
      if (progressed) {
        t_idle = 0;
        spins = 0;
      } else if ((++spins & 255u) == 0) {
        // bounded like every other wait: give up after WAIT_LIMIT_NS without progress
        const uint64_t now = ptx::globaltimer_ns();
        if (t_idle == 0) t_idle = now;
        if (*ab.flag || now - t_idle > WAIT_LIMIT_NS || spins >= WAIT_MAX_ITERS) {
          if (!*ab.flag) {
            *ab.flag = 1u;
            ptx::st_cluster_u32(ab.peer, 1u);
            atomicOr(&g_fa_error, ERR_WAIT_MMA);
          }
          ok = false;
          break;
        }
      }
    }
    if (!ok) break;
    kv_base += 2 * n;
    ++unit_it;
  }
  // every product this warp issued has finished before tensor memory is freed
  ptx::mma2_commit_elect(bar.drain());
  drain_wait(bar.drain(), 0);
}

// ---------------------------------------------------------------------------- softmax

// Maximum of a 128-score row: per 32 columns a tree of three-input maxima (depth 4; a
// chain of them would be 16 deep), then across the four.
__device__ __forceinline__ float row_max128(const uint32_t (&sr)[4][32]) {
  float m[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float t[11];
#pragma unroll
    for (int i = 0; i < 10; ++i)
      t[i] = ptx::max3(__uint_as_float(sr[c][3 * i]), __uint_as_float(sr[c][3 * i + 1]),
                       __uint_as_float(sr[c][3 * i + 2]));
    t[10] = fmaxf(__uint_as_float(sr[c][30]), __uint_as_float(sr[c][31]));
    const float u0 = ptx::max3(t[0], t[1], t[2]), u1 = ptx::max3(t[3], t[4], t[5]);
    const float u2 = ptx::max3(t[6], t[7], t[8]), u3 = fmaxf(t[9], t[10]);
    m[c] = fmaxf(ptx::max3(u0, u1, u2), u3);
  }
  return fmaxf(ptx::max3(m[0], m[1], m[2]), m[3]);
}

// A 128-score row (sr) -> bf16 numerators at t_p (64 columns); adds the sum of the
// unrounded numerators to le.  NPOLY of every 8 column pairs use the FMA-pipe exponential.
// Per 32 columns: all arguments first, then all exponentials, then the packing and the
// sums, so that the exponentials issue back to back.
template <int NPOLY>
__device__ __forceinline__ void pair_numerators(const uint32_t (&sr)[4][32], float sl2,
                                                float neg_m, uint32_t t_p, float &le) {
  const uint64_t scale2 = ptx::f2_pack(sl2, sl2);
  const uint64_t bias2 = ptx::f2_pack(neg_m, neg_m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float x[32], pe[32];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const uint64_t xx = ptx::f2_fma(
          ptx::f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), scale2, bias2);
      ptx::f2_unpack(xx, x[e], x[e + 1]);
    }
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      if (((e % 16) / 2) < NPOLY) {
        exp2_poly_pair(x[e], x[e + 1], pe[e], pe[e + 1]);
      } else {
        pe[e] = ptx::ex2(x[e]);
        pe[e + 1] = ptx::ex2(x[e + 1]);
      }
    }
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      pk[e / 2] = ptx::pack_bf16x2(pe[e], pe[e + 1]);
      acc[(e / 2) & 3] = ptx::f2_add(acc[(e / 2) & 3], ptx::f2_pack(pe[e], pe[e + 1]));
    }
    ptx::tmem_st16(t_p + c * 16, pk);
  }
  float a0, a1;
  ptx::f2_unpack(ptx::f2_add(ptx::f2_add(acc[0], acc[1]), ptx::f2_add(acc[2], acc[3])), a0, a1);
  le += a0 + a1;
}

template <int D, bool CAUSAL, bool OUT_F32>
__device__ void pair_softmax_role(const FwdParams &p, uint32_t tmem,
                                  const PBars<PCfg<D>::NSLOT> &bar,
                                  volatile uint32_t *ring, const Abort &ab, uint32_t rank,
                                  volatile float *xch, uint8_t *stage) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = warp / 4;        // key stream (blocks j with j mod 2 == h); O dims [64 h, 64 h + 64)
  const int wq = warp % 4;       // TMEM lane quarter
  const int r_cta = wq * 32 + lane;  // row inside the CTA's 128
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t t_s = tmem + lane_base + h * BN;
  using C = PCfg<D>;
  const uint32_t t_o = tmem + lane_base + C::O_COL0;
  const uint32_t t_p = tmem + lane_base + C::p_col(h);
  const uint32_t p_full_c = ptx::mapa(bar.p_full(h), 0);
  const uint32_t s_free_c = ptx::mapa(bar.s_free(h), 0);
  const uint32_t o_empty_c = ptx::mapa(bar.o_empty(), 0);
  const uint32_t my_hand = bar.hand(h, wq), other_hand = bar.hand(h ^ 1, wq);
  const uint32_t xbar = bar.xchg(wq);
  volatile float *mh = xch;            // [stream][row]: maximum in use after its latest block
  volatile float *xl = xch + 2 * BM;   // [stream][row]: row sums, for the epilogue
  volatile float *mx = xch + 4 * BM;   // [stream][row]: exact running maximum (statistics)
  uint32_t n_steps = 0, n_lazy = 0, n_eager = 0;  // rescale statistics of this thread's row
  const float NEG_INF = -__int_as_float(0x7f800000);
  uint32_t sph = 0;        // phase bit of s_full(h)
  uint32_t hph = 0;        // phase bit of the other stream's hand barrier
  uint32_t xph = 0;        // phase bit of xchg
  uint32_t pvc0 = 0, pvc1 = 0;  // P V products committed on pv_done(0 / 1) in earlier units
  uint32_t unit_it = 0, taken = 0;
  // arrive on one of CTA 0's barriers (local in CTA 0, remote from CTA 1)
  auto arrive0 = [&](uint32_t local, uint32_t remote) {
    if (rank == 0)
      ptx::mbar_arrive_elect(local);
    else
      ptx::mbar_arrive_remote_elect(remote);
  };
  // the maximum in use (and the exact running maximum) after the other stream's latest
  // block
  auto take_other_max = [&](float &m, float &me) {
    const bool ok = pwait(other_hand, hph, ab, ERR_WAIT_SOFTMAX);
    hph ^= 1u;
    if (!__all_sync(0xffffffffu, ok)) return false;
    m = mh[(h ^ 1) * BM + r_cta];
    me = mx[(h ^ 1) * BM + r_cta];
    return true;
  };
  // at the end of the work list: add this warp's rescale statistics to the device counters
  auto flush_stats = [&]() {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_steps += __shfl_xor_sync(0xffffffffu, n_steps, o);
      n_lazy += __shfl_xor_sync(0xffffffffu, n_lazy, o);
      n_eager += __shfl_xor_sync(0xffffffffu, n_eager, o);
    }
    if (lane == 0) {
      atomicAdd(&g_fa_rescale_stats[0], static_cast<unsigned long long>(n_steps));
      atomicAdd(&g_fa_rescale_stats[1], static_cast<unsigned long long>(n_lazy));
      atomicAdd(&g_fa_rescale_stats[2], static_cast<unsigned long long>(n_eager));
    }
  };

  for (;;) {
    uint32_t u;
    {
      const int s = taken % UNIT_RING_P;
      const bool ok =
          pwait<true>(bar.unit_full(s), (taken / UNIT_RING_P) & 1u, ab, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      u = ring[s];
      __syncwarp();
      ptx::mbar_arrive_cluster_elect(ptx::mapa(bar.unit_empty(s), 0));
      ++taken;
    }
    if (u >= static_cast<uint32_t>(p.num_units)) {
      flush_stats();
      return;
    }
    const PUnit w = pair_decode<CAUSAL>(p, static_cast<int>(u));
    const int n = w.n;
    const int row0 = w.r0 + static_cast<int>(rank) * BM;  // first row of this CTA
    const int row = row0 + r_cta;
    const float sl2 = p.scale_log2;
    const int key_lim = CAUSAL ? min(row + w.off, p.Nk - 1) : p.Nk - 1;
    float m_used = NEG_INF;  // maximum in use after the latest block this warp knows of
    float m_ref = NEG_INF;   // maximum this stream's sum l is relative to
    float l = 0.f;

    for (int j = h; j < n; j += 2) {
      bool ok = pwait(bar.s_full(h), sph, ab, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      sph ^= 1u;
      ptx::tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld32(t_s + c * 32, sr[c]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::reg_fence32(sr[c]);
      // S(h) is read: the tensor core may compute S(j+2) into it
      ptx::tc_fence_before();
      __syncwarp();
      arrive0(bar.s_free(h), s_free_c);

      const int kv0 = j * BN;
      const bool need_mask = (CAUSAL && kv0 + BN - 1 > row0 + w.off) || (kv0 + BN > p.Nk);
      if (need_mask) {
        const int lim = key_lim - kv0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e > lim) sr[c][e] = __float_as_uint(NEG_INF);
      }
      const float xmax = row_max128(sr) * sl2;
      // the maximum in use before this block, then the one after it, handed on to block j+1
      float m_prev = NEG_INF, me_prev = NEG_INF;
      if (j > 0 && !take_other_max(m_prev, me_prev)) return;
      const float m_new = xmax > m_prev + RESCALE_THRESHOLD ? xmax : m_prev;
      ++n_steps;
      n_lazy += (m_new != m_prev && m_prev != NEG_INF) ? 1u : 0u;
      n_eager += (xmax > me_prev && me_prev != NEG_INF) ? 1u : 0u;
      mx[h * BM + r_cta] = fmaxf(me_prev, xmax);
      mh[h * BM + r_cta] = m_new;
      __syncwarp();
      ptx::mbar_arrive_elect(my_hand);
      m_used = m_new;
      // this stream's sum follows the maximum in use
      if (m_new != m_ref) {
        l = (m_ref == NEG_INF) ? 0.f : l * ptx::ex2(m_ref - m_new);
        m_ref = m_new;
      }
      if (__any_sync(0xffffffffu, m_new != m_prev && j > 0)) {
        // rescale O to the new maximum once P(j-1) V (the other stream's, the last product
        // into O so far) has completed; P(j) V is issued only after this block's p_full
        const int b1 = (j - 1) & 1;
        ok = pwait(bar.pv_done(b1), ((b1 ? pvc1 : pvc0) + (j - 1) / 2) & 1u, ab,
                   ERR_WAIT_SOFTMAX);
        if (!__all_sync(0xffffffffu, ok)) return;
        ptx::tc_fence_after();
        const float alpha = (m_new != m_prev) ? ptx::ex2(m_prev - m_new) : 1.f;
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
      }
      // P(h) was read by this stream's previous product P(j-2) V
      if (j >= 2) {
        ok = pwait(bar.pv_done(h), ((h ? pvc1 : pvc0) + (j - 2) / 2) & 1u, ab, ERR_WAIT_SOFTMAX);
        if (!__all_sync(0xffffffffu, ok)) return;
        ptx::tc_fence_after();
      }
      const float neg_m = (m_new == NEG_INF) ? 0.f : -m_new;
      float le = 0.f;
      if (POLY_PAIRS == 0 || need_mask)
        pair_numerators<0>(sr, sl2, neg_m, t_p, le);
      else
        pair_numerators<POLY_PAIRS>(sr, sl2, neg_m, t_p, le);
      l += le;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      arrive0(bar.p_full(h), p_full_c);
    }

    // Epilogue.  m = the maximum in use after block n-1; O and both sums are relative to it
    // once each stream's sum is brought there: O = O_acc / (l_0 + l_1), LSE = ln 2 (m +
    // log2(l_0 + l_1)).
    {
      float m = m_used, me_unused;
      if (((n - 1) & 1) != h && !take_other_max(m, me_unused)) return;
      const float lm = (l > 0.f) ? l * ptx::ex2(m_ref - m) : 0.f;
      bool ok = pwait(bar.o_full(), unit_it & 1u, ab, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      ptx::tc_fence_after();
      // written only after o_full: the partner has read the previous unit's value, since
      // this unit's products waited for its o_empty
      xl[h * BM + r_cta] = lm;
      __syncwarp();
      ptx::mbar_arrive_elect(xbar);
      ok = pwait(xbar, xph, ab, ERR_WAIT_SOFTMAX);
      xph ^= 1u;
      if (!__all_sync(0xffffffffu, ok)) return;
      const float lt = lm + xl[(h ^ 1) * BM + r_cta];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const bool valid = row < p.Nq;
      const size_t orow = static_cast<size_t>(w.bh) * p.Nq + (valid ? row : 0);
      // O leaves through this warp's staging buffer in shared memory, 64 bytes of each row
      // (32 bf16 or 16 fp32 columns) at a time: each thread writes its row's four 16-byte
      // chunks, XOR-swizzled by row so that the writes meet no bank conflicts, then the warp
      // stores whole 64-byte row segments, 8 rows per instruction, instead of 32 scattered
      // 16-byte pieces.
      constexpr int OB = OUT_F32 ? 4 : 2;   // bytes per output element
      uint8_t *const st = stage + warp * STAGE_WARP_BYTES;
      const int row_w0 = row - lane;        // first row of this warp
      auto put = [&](const uint4(&v)[4], int col) {  // col: first column of the segment
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(st + lane * 64 + (q ^ ((lane >> 1) & 3)) * 16) = v[q];
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = k * 8 + lane / 4, q = lane % 4;
          const uint4 val = *reinterpret_cast<const uint4 *>(st + r * 64 + (q ^ ((r >> 1) & 3)) * 16);
          const int rr = row_w0 + r;
          if (rr < p.Nq)
            *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.o) +
                                       ((static_cast<size_t>(w.bh) * p.Nq + rr) * D + col) * OB +
                                       q * 16) = val;
        }
        __syncwarp();
      };
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const uint32_t col = h * (D / 2) + c * 32;
        uint32_t a[32];
        ptx::tmem_ld32(t_o + col, a);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(a);
        if (OUT_F32) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t *s4 = a + 16 * half + 4 * q;
              v[q] = make_uint4(__float_as_uint(__uint_as_float(s4[0]) * inv),
                                __float_as_uint(__uint_as_float(s4[1]) * inv),
                                __float_as_uint(__uint_as_float(s4[2]) * inv),
                                __float_as_uint(__uint_as_float(s4[3]) * inv));
            }
            put(v, col + 16 * half);
          }
        } else {
          uint32_t hh[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            hh[e] = ptx::pack_bf16x2(__uint_as_float(a[2 * e]) * inv, __uint_as_float(a[2 * e + 1]) * inv);
          uint4 v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) v[q] = make_uint4(hh[4 * q], hh[4 * q + 1], hh[4 * q + 2], hh[4 * q + 3]);
          put(v, col);
        }
      }
      if (valid && h == 0)
        p.lse[orow] = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994530942f : NEG_INF;
      ptx::tc_fence_before();
      __syncwarp();
      arrive0(bar.o_empty(), o_empty_c);
    }
    pvc0 += (n + 1) / 2;
    pvc1 += n / 2;
    ++unit_it;
  }
}

// ---------------------------------------------------------------------------- kernel

template <int D, bool CAUSAL, bool OUT_F32>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t smem = (raw + 1023u) & ~1023u;  // 1024-aligned for 128-byte swizzle
  uint8_t *smem_gen = smem_raw + (smem - raw);
  using C = PCfg<D>;
  const PBars<C::NSLOT> bar{smem + C::BAR_OFF};
  uint32_t *ctl = reinterpret_cast<uint32_t *>(smem_gen + C::CTL_OFF);
  volatile uint32_t *tmem_slot = ctl;
  volatile uint32_t *abort_flag = ctl + 1;
  volatile uint32_t *ring = ctl + 4;
  volatile float *xch = reinterpret_cast<volatile float *>(smem_gen + C::XCH_OFF);
  const uint32_t rank = ptx::cluster_ctarank();
  const Abort ab{abort_flag, ptx::mapa(ptx::smem_addr(ctl + 1), rank ^ 1u)};

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      ptx::mbar_init(bar.slot_full(s), 1);
      ptx::mbar_init(bar.slot_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar.q_full(b), 1);
      ptx::mbar_init(bar.q_empty(b), 1);
      ptx::mbar_init(bar.s_full(b), 1);
      ptx::mbar_init(bar.s_free(b), STREAM_WARPS_PAIR);
      ptx::mbar_init(bar.p_full(b), STREAM_WARPS_PAIR);
      ptx::mbar_init(bar.pv_done(b), 1);
    }
    ptx::mbar_init(bar.o_full(), 1);
    ptx::mbar_init(bar.o_empty(), SOFTMAX_WARPS_PAIR);
    ptx::mbar_init(bar.drain(), 1);
    for (int wq = 0; wq < 4; ++wq) {
      ptx::mbar_init(bar.xchg(wq), 2);        // warps wq and wq + 4
      ptx::mbar_init(bar.hand(0, wq), 1);     // one publishing warp per block
      ptx::mbar_init(bar.hand(1, wq), 1);
    }
    for (int s = 0; s < UNIT_RING_P; ++s) {
      ptx::mbar_init(bar.unit_full(s), 1);
      ptx::mbar_init(bar.unit_empty(s), UNIT_CONSUMERS);
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    ptx::tmem_alloc_pair(ptx::smem_addr(ctl), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialised and the pair's tensor memory allocated before
  // either CTA signals the other
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8)
    ptx::setmaxnreg_inc<SOFTMAX_REGS>();
  else
    ptx::setmaxnreg_dec<OTHER_REGS>();

  if (warp < 8) {
    pair_softmax_role<D, CAUSAL, OUT_F32>(p, tmem, bar, ring, ab, rank, xch, smem_gen + C::STAGE_OFF);
  } else if (rank == 0 && warp == MMA_WARP) {
    pair_mma_role<D, CAUSAL>(p, smem, tmem, bar, ring, ab);
    __syncwarp();
  } else if (warp == TMA_WARP) {
    if (lane == 0) pair_load_role<D, CAUSAL>(&tmQ, &tmK, &tmV, p, smem, bar, ring, ab, rank);
    __syncwarp();
  }

  // neither CTA leaves (or frees the pair's tensor memory) while the other may still
  // signal it or run products on it
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
  }
}

}  // namespace pair
}  // namespace fa
