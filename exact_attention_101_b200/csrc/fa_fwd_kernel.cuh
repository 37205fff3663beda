// fa_fwd_kernel.cuh -- fused exact-attention forward kernel for B200 (sm_100a).
//
// One persistent CTA per SM claims work units from a list shared by the launch (see
// "Work distribution" below).  A unit is 256 query rows (two 128-row Q tiles) of one
// (batch, query head); the two tiles share every K/V tile that is streamed through
// shared memory.  The method is the IO-aware tiled
// attention of the page "FlashAttention (DE)" (sections "Tiling und blockweise
// Verarbeitung", "Online-Softmax-Berechnung", "Zusammenfassen von Operationen in einem
// CUDA-Kernel"): S = Q K^T, the mask, the online softmax and O += P V all happen on chip;
// only O and the per-row log-sum-exp are written.  The warp roles follow the idea of a
// warp-specialised pipeline (page "FlashAttention 4: Praxisleitfaden ...", section "Was
// ist neu in FlashAttention 4?": loading, MMA, softmax, rescaling, epilogue), mapped
// onto sm_100a as follows:
//
//   warps 0-3   softmax + epilogue for Q tile 0 (one thread per query row)
//   warps 4-7   softmax + epilogue for Q tile 1
//   warp  8     tensor-memory allocator; tcgen05.mma issuer for Q tile 0
//   warp  9     TMA producer (one lane)
//   warp  10    tcgen05.mma issuer for Q tile 1
//   warp  11    idle (it completes the third warpgroup)
// A unit is NT = 2 Q tiles (256 query rows) for head dims 64 and 128.  At head dim 256 a
// second tile fits neither in tensor memory (two 256-column O accumulators) nor next to a
// useful K/V ring in shared memory, so a unit is one Q tile (NT = 1) and warps 4-7 and 10
// stay idle.
//
// Key tiles are BN = 64 keys, and every Q tile has NBUF = 2 score buffers in tensor
// memory: while the softmax warps of a tile turn S(j) into P(j), the tensor core already
// computes S(j+1), and S(j+NBUF) as soon as P(j) has been consumed.  So a tile's softmax
// never waits for its own P.V product, and the two tiles' softmax warps -- one of each
// per SM sub-partition -- can both be busy at once.  This matters on B200 because, at head dim 128, the
// exponentials of one score tile take the SFU as long as the tensor core takes for that
// tile's two products.
//
// Tensor memory (512 columns x 128 lanes x 32 bit), BN = 64:
//   S(x, b) at x*NBUF*64 + b*64, 64 fp32 columns (tile x, buffer b); the numerators P of
//   that buffer (bf16 pairs or e4m3 quads packed in 32-bit columns) overwrite its upper
//   32 columns; O_x accumulator at O_COL0 + x*D (O_COL0 = 256).
//
// Registers: the kernel is launched with LAUNCH_REGS per thread (384 threads); the third
// warpgroup gives registers back (setmaxnreg.dec to OTHER_REGS) and the two softmax
// warpgroups take them (setmaxnreg.inc to SOFTMAX_REGS).  256*SOFTMAX_REGS +
// 128*OTHER_REGS stays within the launch pool 384*LAUNCH_REGS; the host refuses to launch
// a build whose register count would make that sum exceed the pool.
//
// Shared memory: Q0, Q1 (128-row tiles) and a ring of NSLOT 64-row K/V tiles, all in the
// 128-byte swizzled layout that TMA writes and the tensor core reads; the mbarriers.
//
// Synchronisation (all mbarriers):
//   q_full / q_empty        Q tiles of a unit loaded / no longer read by an MMA
//   slot_full / slot_empty  ring slot loaded (TMA tx bytes) / released by an MMA commit
//   s_full[x][b]            S(x, b) computed
//   p_full[x][b]            P(x, b) written by the 128 softmax threads of tile x
//   pv_done[x][n & 1]       P.V product n of tile x finished (for the rare rescale)
//   o_full[x] / o_empty[x]  O_x final for the unit / read out by the epilogue
//
// MMA order of tile x inside a unit (j = key tile): S(x, 0) .. S(x, NBUF-1), then for
// every j PV(x, j), S(x, j+NBUF).  S(x, j+NBUF) reuses the buffer of P(x, j) and is issued after
// PV(x, j) by the same thread: tcgen05 operations from one thread run in issue order, so
// the product reads P before the next scores overwrite it.
//
// Softmax details.  Scores are moved into the base-2 domain with one FFMA,
// x = s * (scale * log2 e), and p = 2^(x - m_used).  m_used is only raised when a key
// tile's row maximum exceeds it by more than RESCALE_THRESHOLD (lazy rescaling, page
// "FlashAttention 4: Praxisleitfaden ...", section "Intelligenteres Online-Softmax-
// Rescaling in FA4"), so p <= 2^RESCALE_THRESHOLD and the accumulator O and the sums are
// multiplied by 2^(m_old - m_new) only then.  The causal mask is applied only on key
// tiles that cross the diagonal; tiles entirely above it are never loaded.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fa {

// ---------------------------------------------------------------------------- config

constexpr int BM = 128;               // query rows per Q tile (MMA M)
constexpr int BN = 64;                // keys per K/V tile (MMA N of S = Q K^T)
constexpr int UNIT_ROWS = 2 * BM;     // query rows per work unit
constexpr int NUM_THREADS = 384;
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
constexpr int LAUNCH_REGS = 168;    // 65536 / 384, rounded down to a multiple of 8
#ifndef FA_SOFTMAX_REGS
#define FA_SOFTMAX_REGS 200
#endif
constexpr int SOFTMAX_REGS = FA_SOFTMAX_REGS;
constexpr int OTHER_REGS = (NUM_THREADS * LAUNCH_REGS - 256 * SOFTMAX_REGS) / 128 / 8 * 8;
static_assert(OTHER_REGS >= 64, "register split leaves too few for the MMA/TMA warps");
static_assert(256 * SOFTMAX_REGS + 128 * OTHER_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch pool");
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units: p <= 256
#ifndef FA_EXP2_POLY_PAIRS
#define FA_EXP2_POLY_PAIRS 0
#endif
#ifndef FA_EXP2_POLY_PAIRS_FP8
#define FA_EXP2_POLY_PAIRS_FP8 2
#endif
// Column pairs (of every 8) whose exponentials use the FMA-pipe polynomial on unmasked
// tiles; the rest use the MUFU unit.  bf16: none (every share measured slower, at d = 64
// by 13 % and more).  e4m3: its products take half the tensor time of bf16, so the SFU
// leads by two to one; two pairs of eight measured 2.5 % faster (B8 H16 N4096 d128), and P
// is rounded to e4m3 anyway, far coarser than the polynomial's 7.5e-5.
constexpr int EXP2_POLY_PAIRS = FA_EXP2_POLY_PAIRS;
constexpr int EXP2_POLY_PAIRS_FP8 = FA_EXP2_POLY_PAIRS_FP8;
static_assert(EXP2_POLY_PAIRS >= 0 && EXP2_POLY_PAIRS <= 8, "pairs per 16-column chunk");
static_assert(EXP2_POLY_PAIRS_FP8 >= 0 && EXP2_POLY_PAIRS_FP8 <= 8, "pairs per 16-column chunk");
#ifndef FA_D64_SCORE_BUFFERS
#define FA_D64_SCORE_BUFFERS 2   // score buffers per Q tile at head dim 64 (2 or 3)
#endif

// Error bits written to the device error word when a bounded wait runs out.
constexpr uint32_t ERR_WAIT_SOFTMAX = 1u << 0;
constexpr uint32_t ERR_WAIT_MMA = 1u << 1;
constexpr uint32_t ERR_WAIT_LOAD = 1u << 2;
constexpr uint32_t ERR_WAIT_DRAIN = 1u << 3;
constexpr uint32_t ERR_WAIT_SELFTEST = 1u << 4;

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s per wait

// Work distribution: every CTA starts with unit blockIdx.x; after that its TMA warp claims
// the next unit from a counter shared by the launch (one atomic per unit), so CTAs that
// drew short units (causal, variable lengths) take more of them.  Each launch owns one
// slot of g_fa_sched, chosen round-robin by the host: word 0 counts the units claimed,
// word 1 the CTAs that have finished; the last CTA to finish sets both back to zero for
// the slot's next launch.  (Launches that share a slot while both are in flight would
// share the counter: the host cycles through SCHED_SLOTS slots per device.)
constexpr int SCHED_SLOTS = 4096;
__device__ unsigned int g_fa_sched[SCHED_SLOTS][2];
constexpr int UNIT_RING = 4;  // units the TMA warp publishes ahead to the consumer warps
constexpr uint32_t WAIT_MAX_ITERS = 1u << 28;

template <int D, bool FP8>
struct TileCfg {
  static constexpr int NT = D > 128 ? 1 : 2;         // Q tiles per unit
  static constexpr int UNIT = NT * BM;               // query rows per unit
  static constexpr int ELEM = FP8 ? 1 : 2;           // bytes per element
  static constexpr int ROW_BYTES = D * ELEM;         // bytes per tile row
  static_assert(ROW_BYTES % 128 == 0, "tile rows must be whole 128-byte swizzle rows");
  static constexpr int NBOX = ROW_BYTES / 128;       // 128-byte-wide TMA boxes per row
  static constexpr int BOX_ELEMS = 128 / ELEM;       // elements per box row
  static constexpr int Q_BOX_BYTES = BM * 128;       // 128 rows x 128 bytes
  static constexpr int KV_BOX_BYTES = BN * 128;      // 64 rows x 128 bytes
  static constexpr int Q_TILE_BYTES = NBOX * Q_BOX_BYTES;
  static constexpr int KV_TILE_BYTES = NBOX * KV_BOX_BYTES;
  static constexpr int NSLOT = 131072 / KV_TILE_BYTES;  // 128 KB ring: 4, 8 or 16 slots
  static_assert((NSLOT & (NSLOT - 1)) == 0, "ring size must be a power of two");
  static constexpr int MMA_K = FP8 ? 32 : 16;        // K extent of one MMA instruction
  static constexpr int S_KSTEPS = D / MMA_K;         // MMAs per S = Q K^T
  static constexpr int PV_KSTEPS = BN / MMA_K;       // MMAs per O += P V
  static constexpr uint32_t AB_FORMAT = FP8 ? 0u : 1u;  // e4m3 : bf16
  static constexpr uint32_t IDESC_S = ptx::make_idesc(AB_FORMAT, BM, BN, 0);
  static constexpr uint32_t IDESC_O = ptx::make_idesc(AB_FORMAT, BM, D, 1);
  // TMEM column map.  Score buffers per Q tile: two; at D = 64 tensor memory also holds a
  // third next to the two O accumulators (FA_D64_SCORE_BUFFERS = 3).  With S(j) issued
  // after P.V(j-NBUF), up to NBUF-1 products may be outstanding when the softmax of key
  // tile j rescales, so P.V product n commits to pv_done(x, n & 1): each of the two
  // barriers then has at most one pending phase at that point, and a parity wait on it is
  // exact for either count.  The third buffer passes parity but measured 0.7 % (non-causal)
  // and 1.3 % (causal) slower at B 16, H 12, N 2048 on B200, so two is the default.
  static constexpr int NBUF = D == 64 ? FA_D64_SCORE_BUFFERS : 2;
  static_assert(NBUF == 2 || NBUF == 3, "two or three score buffers per Q tile");
  static constexpr uint32_t S_COLS = NBUF * 64;          // score columns of one Q tile
  __host__ __device__ static constexpr uint32_t s_col(int x, int b) { return x * S_COLS + b * 64; }
  static constexpr uint32_t P_OFF = 32;                  // P inside a 64-column S buffer
  static constexpr uint32_t O_COL0 = NT * S_COLS > 256 ? NT * S_COLS : 256, O_COL1 = O_COL0 + D;
  static_assert(O_COL0 + NT * D <= TMEM_COLS, "TMEM budget");
  // Shared memory map (offsets from a 1024-aligned base).
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NT * Q_TILE_BYTES;
  // epilogue staging: 32 rows x 32 fp32 columns per softmax warp
  static constexpr int STAGE_WARP_BYTES = 32 * 32 * 4;
  static constexpr int STAGE_OFF = RING_OFF + NSLOT * KV_TILE_BYTES;
  static constexpr int BAR_OFF = STAGE_OFF + 4 * NT * STAGE_WARP_BYTES;
  static constexpr int NUM_BARS = 2 * NSLOT + 24 + 2 * UNIT_RING;
  static constexpr int CTL_OFF = BAR_OFF + NUM_BARS * 8;
  // control words: TMEM base, abort flag, 2 spare, then the ring of published units
  static constexpr int SMEM_BYTES = 1024 + CTL_OFF + 16 + 4 * UNIT_RING;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};


struct FwdParams {
  void *o;
  float *lse;
  const float *descale_q;  // fp8 only: [B*Hq]
  const float *descale_k;  // fp8 only: [B*Hkv]
  const float *descale_v;  // fp8 only: [B*Hkv]
  const int *cu_q;         // varlen only: [B+1] first token of each query sequence
  const int *cu_k;         // varlen only: [B+1] first token of each key sequence
  int B, Hq, Hkv, Nq, Nk;  // varlen: Nq, Nk = total tokens of the packed Q and K tensors
  int group;        // Hq / Hkv
  int num_qb;       // ceil(Nq / unit rows); varlen: ceil(longest query sequence / unit rows)
  int num_units;    // B * Hq * num_qb
  float scale_log2; // softmax scale * log2(e)
  // dropout (kernels instantiated with DROPOUT only): key j of query row i of (batch,
  // head) bh is kept iff byte j mod 32 of the Philox4x64-10 block for counter
  // (j / 32, i, bh, 0) and key (seed, offset) is >= drop_thr; kept weights are scaled by
  // keep_scale = 1 / (1 - drop_thr / 256)
  uint64_t seed, offset;
  uint32_t drop_thr4;  // drop_thr in every byte
  float keep_scale;
  unsigned int *sched;  // this launch's slot of g_fa_sched (two words, zero at launch)
};

struct Unit {
  int bh;     // b * Hq + hq
  int bhk;    // b * Hkv + hq / group
  int qh, kh; // head coordinate of the Q and K/V tensor maps (bh, bhk; varlen: hq, hk)
  int q_tok;  // varlen: token of the sequence's first query in the packed tensor (else 0)
  int k_tok;  // varlen: token of the sequence's first key (else 0)
  int len_q;  // queries of the sequence (Nq for fixed length)
  int len_k;  // keys of the sequence (Nk)
  int off;    // causal diagonal: query i sees keys j <= i + off (off = len_k - len_q)
  int r0;     // first query row of the unit, within its sequence
  int n0;     // key tiles visited by Q tile 0 (at least 1)
  int n1;     // key tiles visited by Q tile 1 (>= n0)
  bool empty; // varlen: the unit starts past the end of its sequence
};

// Key tiles that query rows up to `last_row` visit: all of them, or under the causal mask
// those up to the diagonal.  At least one, so that a row without admissible keys still
// runs through the pipeline (its scores are all masked and it gets O = 0, LSE = -inf).
template <bool CAUSAL>
__device__ __forceinline__ int key_tiles(int last_row, int len_k, int off) {
  const int last_key = CAUSAL ? min(len_k - 1, last_row + off) : len_k - 1;
  return last_key < 0 ? 1 : last_key / BN + 1;
}

// Work list: groups of consecutive (batch, query head) pairs, so that the CTAs running at
// the same time share the K/V of a few heads in L2 (and query heads that share a K/V head
// are neighbours).  Inside a group the query blocks run last-first across its heads.
// Under the causal mask that is longest-first over CAUSAL_HEAD_GROUP heads, so that the
// units claimed last, at the end of the list, are short ones.  Without the mask every
// unit costs the same and a group is one head: fewer heads in flight read less K/V from
// DRAM (8 heads of 8 MB each did not stay in L2).  With variable lengths every sequence
// gets num_qb blocks (those of the longest sequence); the blocks past the end of a
// shorter sequence are empty and never published.
constexpr int CAUSAL_HEAD_GROUP = 8;

template <bool CAUSAL, bool VARLEN, int UNIT = UNIT_ROWS>
__device__ __forceinline__ Unit decode_unit(const FwdParams &p, int u) {
  constexpr int HG = CAUSAL ? CAUSAL_HEAD_GROUP : 1;
  const int BH = p.num_units / p.num_qb;      // (batch, query head) pairs
  const int g = u / (HG * p.num_qb);          // head group
  const int r = u - g * HG * p.num_qb;
  const int heads = min(HG, BH - g * HG);     // the last group may be smaller
  const int qb = p.num_qb - 1 - r / heads;
  Unit w;
  w.bh = g * HG + r % heads;
  const int b = w.bh / p.Hq, hq = w.bh % p.Hq;
  w.bhk = b * p.Hkv + hq / p.group;
  w.r0 = qb * UNIT;
  if (VARLEN) {
    w.qh = hq;
    w.kh = hq / p.group;
    w.q_tok = p.cu_q[b];
    w.k_tok = p.cu_k[b];
    w.len_q = p.cu_q[b + 1] - w.q_tok;
    w.len_k = p.cu_k[b + 1] - w.k_tok;
  } else {
    w.qh = w.bh;
    w.kh = w.bhk;
    w.q_tok = 0;
    w.k_tok = 0;
    w.len_q = p.Nq;
    w.len_k = p.Nk;
  }
  w.empty = VARLEN && w.r0 >= w.len_q;
  w.off = w.len_k - w.len_q;
  w.n0 = key_tiles<CAUSAL>(w.r0 + BM - 1, w.len_k, w.off);
  // with one Q tile per unit there is no tile 1: the ring holds tile 0's key tiles only
  w.n1 = UNIT > BM ? key_tiles<CAUSAL>(w.r0 + 2 * BM - 1, w.len_k, w.off) : w.n0;
  return w;
}

__device__ unsigned int g_fa_error = 0;

// Counters of the online softmax's rescaling, summed over the launches of the CTA-pair
// forward (read and cleared by fa_rescale_stats): [0] (query row, key block) steps, [1]
// rescales of the accumulator under the lazy rule the kernel runs, [2] rescales the eager
// rule -- move the maximum whenever a block raises it -- would have made on the same rows.
// A rescale is counted only once the row has seen an admissible key.
__device__ unsigned long long g_fa_rescale_stats[3];

// Bounded wait on an mbarrier phase.  Returns false if another warp of the CTA aborted or
// if this wait ran out (then it raises the CTA abort flag and the device error word).
__device__ __forceinline__ bool wait_phase_slow(uint32_t bar, uint32_t parity,
                                                volatile uint32_t *abort_flag, uint32_t who,
                                                uint64_t limit_ns = WAIT_LIMIT_NS) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1; it < WAIT_MAX_ITERS; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > limit_ns) break;
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
  // three score buffers reserved per Q tile (TileCfg::NBUF of them used)
  __device__ uint32_t s_full(int x, int b) const { return base + 8u * (2 * NSLOT + 2 + 3 * x + b); }
  __device__ uint32_t p_full(int x, int b) const { return base + 8u * (2 * NSLOT + 8 + 3 * x + b); }
  // P.V product n of tile x commits to pv_done(x, n & 1)
  __device__ uint32_t pv_done(int x, int q) const { return base + 8u * (2 * NSLOT + 14 + 2 * x + q); }
  __device__ uint32_t o_full(int x) const { return base + 8u * (2 * NSLOT + 18 + x); }
  __device__ uint32_t o_empty(int x) const { return base + 8u * (2 * NSLOT + 20 + x); }
  __device__ uint32_t drain(int x) const { return base + 8u * (2 * NSLOT + 22 + x); }
  // ring of published work units: written (full) by the TMA warp, read (empty) by the
  // MMA and softmax warps
  __device__ uint32_t unit_full(int s) const { return base + 8u * (2 * NSLOT + 24 + s); }
  __device__ uint32_t unit_empty(int s) const {
    return base + 8u * (2 * NSLOT + 24 + UNIT_RING + s);
  }
};

// The next work unit for a consumer warp (all 32 lanes): the one the TMA warp published
// at ring position `taken`; a value >= num_units ends the list.  False if the wait was
// aborted or ran out.
template <class BarsT>
__device__ __forceinline__ bool take_unit(const BarsT &bar, volatile uint32_t *ring,
                                          uint32_t &taken, volatile uint32_t *abort_flag,
                                          uint32_t who, uint32_t &u) {
  const int s = taken % UNIT_RING;
  const bool ok = wait_phase(bar.unit_full(s), (taken / UNIT_RING) & 1u, abort_flag, who);
  if (!__all_sync(0xffffffffu, ok)) return false;
  u = ring[s];
  __syncwarp();
  ptx::mbar_arrive_elect(bar.unit_empty(s));
  ++taken;
  return true;
}

// ---------------------------------------------------------------------------- producer

template <int D, bool CAUSAL, bool FP8, bool VARLEN>
__device__ void load_role(const CUtensorMap *tmQ, const CUtensorMap *tmK, const CUtensorMap *tmV,
                          const FwdParams &p, uint32_t smem, const Bars<TileCfg<D, FP8>::NSLOT> &bar,
                          volatile uint32_t *unit_ring, volatile uint32_t *abort_flag) {
  using C = TileCfg<D, FP8>;
  ptx::prefetch_tmap(tmQ);
  ptx::prefetch_tmap(tmK);
  ptx::prefetch_tmap(tmV);
  uint32_t issued = 0;     // K/V slot loads issued so far
  uint32_t q_issued = 0;   // Q loads issued so far
  uint32_t published = 0;  // units published to the consumer warps
  const uint32_t num_units = static_cast<uint32_t>(p.num_units);
  auto claim = [&]() { return gridDim.x + atomicAdd(p.sched, 1u); };
  for (uint32_t u = blockIdx.x;; u = claim()) {
    Unit w;
    if (u < num_units) {
      w = decode_unit<CAUSAL, VARLEN, C::UNIT>(p, static_cast<int>(u));
      if (VARLEN && w.empty) continue;  // past the end of its sequence: never published
    }
    {  // publish u (or, past the last unit, the end of the list)
      const int s = published % UNIT_RING;
      if (!wait_phase(bar.unit_empty(s), ((published / UNIT_RING) & 1u) ^ 1u, abort_flag,
                      ERR_WAIT_LOAD))
        goto drain;
      unit_ring[s] = u;
      ptx::mbar_arrive(bar.unit_full(s));
      ++published;
    }
    if (u >= num_units) break;
    if (!wait_phase(bar.q_empty(), (q_issued & 1u) ^ 1u, abort_flag, ERR_WAIT_LOAD)) goto drain;
    ptx::mbar_arrive_expect_tx(bar.q_full(), C::NT * C::Q_TILE_BYTES);
#pragma unroll
    for (int x = 0; x < C::NT; ++x)
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx)
        // fixed length: map {d, rows, heads}; packed varlen: map {d, heads, tokens}
        ptx::tma_load_3d(smem + C::Q_OFF + x * C::Q_TILE_BYTES + bx * C::Q_BOX_BYTES, tmQ,
                         bar.q_full(), bx * C::BOX_ELEMS,
                         VARLEN ? w.qh : w.r0 + x * BM, VARLEN ? w.q_tok + w.r0 + x * BM : w.qh);
    ++q_issued;
    for (int j = 0; j < w.n1; ++j) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {  // K_j, then V_j
        const int s = issued % C::NSLOT;
        const uint32_t ph = (issued / C::NSLOT) & 1u;
        if (!wait_phase(bar.slot_empty(s), ph ^ 1u, abort_flag, ERR_WAIT_LOAD)) goto drain;
        ptx::mbar_arrive_expect_tx(bar.slot_full(s), C::KV_TILE_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          ptx::tma_load_3d(smem + C::RING_OFF + s * C::KV_TILE_BYTES + bx * C::KV_BOX_BYTES,
                           t ? tmV : tmK, bar.slot_full(s), bx * C::BOX_ELEMS,
                           VARLEN ? w.kh : j * BN, VARLEN ? w.k_tok + j * BN : w.kh);
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

// The start-address field of a descriptor is bits [0,14) of (address >> 4); shared
// memory addresses stay below 2^18, so advancing a descriptor by b bytes is adding b >> 4.
// The issue loops below are fully unrolled with compile-time offsets and run on the whole
// MMA warp (one elected lane issues): the tensor core then gets a new MMA every few
// cycles, which a loop with per-step descriptor arithmetic in one thread cannot sustain.
template <int D, bool FP8>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint64_t q_desc, uint64_t k_desc) {
  using C = TileCfg<D, FP8>;
#pragma unroll
  for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
    constexpr uint32_t step = C::MMA_K * C::ELEM;  // bytes along the head dim per MMA
    const uint32_t kb = kk * step;
    const uint32_t qoff = ((kb / 128) * C::Q_BOX_BYTES + (kb % 128)) >> 4;
    const uint32_t koff = ((kb / 128) * C::KV_BOX_BYTES + (kb % 128)) >> 4;
    if (FP8)
      ptx::mma_f8_ss_elect(tmem_s, q_desc + qoff, k_desc + koff, C::IDESC_S, kk > 0 ? 1u : 0u);
    else
      ptx::mma_bf16_ss_elect(tmem_s, q_desc + qoff, k_desc + koff, C::IDESC_S, kk > 0 ? 1u : 0u);
  }
}

template <int D, bool FP8>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t v_desc,
                                         uint32_t accumulate) {
  using C = TileCfg<D, FP8>;
  // V is [keys x D] with D contiguous: MN-major B operand.  MMA_K key rows of 128 bytes
  // per step; successive 128-byte D chunks are one TMA box apart (the LBO of v_desc).
#pragma unroll
  for (int kk = 0; kk < C::PV_KSTEPS; ++kk) {
    const uint32_t off = (kk * C::MMA_K * 128) >> 4;
    const uint32_t a = tmem_p + kk * 8;  // 8 TMEM columns hold MMA_K packed P values
    const uint32_t acc = kk > 0 ? 1u : accumulate;
    if (FP8)
      ptx::mma_f8_ts_elect(tmem_o, a, v_desc + off, C::IDESC_O, acc);
    else
      ptx::mma_bf16_ts_elect(tmem_o, a, v_desc + off, C::IDESC_O, acc);
  }
}

// One MMA warp per Q tile x (warp 8 for tile 0, warp 10 for tile 1), so that each tile's
// chain P(x, j) -> PV(x, j) -> S(x, j+NBUF) waits only for its own softmax warps while the
// other warp keeps the tensor core busy.  Runs on all 32 lanes of the warp; waits are
// polled by every lane and made warp-uniform, MMAs and commits are issued by one elected
// lane.  K/V ring slots and the Q tiles are shared by the two tiles: each is released by
// two arrivals, one per tile.  Key tiles that only tile 1 visits (causal) get tile 0's
// arrival from tile 1's warp as a plain arrive; it happens only after the slot's load has
// landed, so it can never complete the slot's previous phase early.
template <int D, bool CAUSAL, bool FP8, bool VARLEN>
__device__ void mma_role(const FwdParams &p, uint32_t smem, uint32_t tmem,
                         const Bars<TileCfg<D, FP8>::NSLOT> &bar, const int x,
                         volatile uint32_t *unit_ring, volatile uint32_t *abort_flag) {
  using C = TileCfg<D, FP8>;
  const uint64_t q_d = ptx::smem_desc_sw128(smem + C::Q_OFF + x * C::Q_TILE_BYTES, 16, 1024);
  const uint64_t k_d0 = ptx::smem_desc_sw128(smem + C::RING_OFF, 16, 1024);
  const uint64_t v_d0 = ptx::smem_desc_sw128(smem + C::RING_OFF, C::KV_BOX_BYTES, 1024);
  constexpr uint32_t SLOT_STEP = C::KV_TILE_BYTES >> 4;
  const uint32_t t_o = tmem + (x ? C::O_COL1 : C::O_COL0);
  uint32_t kv_base = 0;
  uint32_t pvn = 0;  // P.V products this warp has issued (all units)
  uint32_t pph = 0;  // phase bits of p_full(x, b), bit b
  uint32_t unit_it = 0;
  auto wait = [&](uint32_t b, uint32_t parity) {
    const bool ok = wait_phase(b, parity, abort_flag, ERR_WAIT_MMA);
    return __all_sync(0xffffffffu, ok);
  };
  auto wait_slot = [&](uint32_t idx) {
    return wait(bar.slot_full(idx % C::NSLOT), (idx / C::NSLOT) & 1u);
  };
  // Release ring slot idx for this tile (and for tile 0 if tile 0 does not visit it).
  auto release = [&](uint32_t idx, bool also_tile0) {
    ptx::mma_commit_elect(bar.slot_empty(idx % C::NSLOT));
    if (also_tile0) ptx::mbar_arrive_elect(bar.slot_empty(idx % C::NSLOT));
  };
  auto scores = [&](const Unit &w, int nx, int j, uint32_t ki) {
    issue_s<D, FP8>(tmem + C::s_col(x, j % C::NBUF), q_d, k_d0 + (ki % C::NSLOT) * SLOT_STEP);
    ptx::mma_commit_elect(bar.s_full(x, j % C::NBUF));
    release(ki, x == 1 && j >= w.n0);
    if (j == nx - 1) ptx::mma_commit_elect(bar.q_empty());
  };
  uint32_t taken = 0;
  for (;;) {
    uint32_t u;
    if (!take_unit(bar, unit_ring, taken, abort_flag, ERR_WAIT_MMA, u) ||
        u >= static_cast<uint32_t>(p.num_units))
      break;
    const Unit w = decode_unit<CAUSAL, VARLEN, C::UNIT>(p, static_cast<int>(u));
    const int nx = x ? w.n1 : w.n0;
    if (!wait(bar.q_full(), unit_it & 1u)) break;
    bool ok = true;
    for (int j = 0; j < C::NBUF && j < nx; ++j) {
      if (!wait_slot(kv_base + 2 * j)) { ok = false; break; }
      ptx::tc_fence_after();
      scores(w, nx, j, kv_base + 2 * j);
    }
    for (int j = 0; j < nx && ok; ++j) {
      const int b = j % C::NBUF;
      const uint32_t vi = kv_base + 2 * j + 1;    // V_j
      if (!wait_slot(vi)) { ok = false; break; }
      if (!wait(bar.p_full(x, b), (pph >> b) & 1u)) { ok = false; break; }
      pph ^= 1u << b;
      if (j == 0 && !wait(bar.o_empty(x), (unit_it & 1u) ^ 1u)) { ok = false; break; }
      ptx::tc_fence_after();
      issue_pv<D, FP8>(t_o, tmem + C::s_col(x, b) + C::P_OFF, v_d0 + (vi % C::NSLOT) * SLOT_STEP,
                       j > 0 ? 1u : 0u);
      ptx::mma_commit_elect(bar.pv_done(x, pvn & 1u));
      ++pvn;
      release(vi, x == 1 && j >= w.n0);
      if (j == nx - 1) ptx::mma_commit_elect(bar.o_full(x));
      if (j + C::NBUF < nx) {
        const uint32_t ki = kv_base + 2 * (j + C::NBUF);  // K_{j+NBUF}, into P(j)'s buffer
        if (!wait_slot(ki)) { ok = false; break; }
        ptx::tc_fence_after();
        scores(w, nx, j + C::NBUF, ki);
      }
    }
    if (!ok) break;
    kv_base += 2 * w.n1;
    ++unit_it;
  }
  // Wait until every MMA issued by this warp has finished before TMEM is freed.
  ptx::mma_commit_elect(bar.drain(x));
  drain_wait(bar.drain(x), 0);
}

// ---------------------------------------------------------------------------- softmax

// Software 2^x for a pair of arguments on the FMA pipe: j = round(x) through the
// 1.5*2^23 addition trick, f = x - j in [-1/2, 1/2], 2^f from the minimax cubic fitted by
// gen_exp2_poly.py (max relative error 7.5e-5, below bf16 and e4m3 rounding), and 2^j
// applied by adding j to the exponent field.  Arguments are clamped at -126 so that the
// exponent stays in range (the result is then below 2^-125, i.e. nothing next to the row
// maximum's term >= 1).  This is the FMA-unit exponential of the page "FlashAttention 4:
// Praxisleitfaden ...", section "Software-Exponentialfunktionen ueber CUDA-Kerne".
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float &y0, float &y1) {
  const float MAGIC = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = ptx::f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = ptx::f2_add(x, ptx::f2_pack(MAGIC, MAGIC));
  const uint64_t jf = ptx::f2_add(t, ptx::f2_pack(-MAGIC, -MAGIC));
  const uint64_t f = ptx::f2_fma(jf, ptx::f2_pack(-1.f, -1.f), x);
  uint64_t q = ptx::f2_fma(f, ptx::f2_pack(5.517166853e-02f, 5.517166853e-02f),
                           ptx::f2_pack(2.426111251e-01f, 2.426111251e-01f));
  q = ptx::f2_fma(q, f, ptx::f2_pack(6.932609677e-01f, 6.932609677e-01f));
  q = ptx::f2_fma(q, f, ptx::f2_pack(9.999280572e-01f, 9.999280572e-01f));
  float t0, t1, q0, q1;
  ptx::f2_unpack(t, t0, t1);
  ptx::f2_unpack(q, q0, q1);
  // low mantissa bits of t hold j (two's complement); shifting them into the exponent
  // field and adding multiplies q by 2^j.
  y0 = __uint_as_float(__float_as_uint(t0) * (1u << 23) + __float_as_uint(q0));
  y1 = __uint_as_float(__float_as_uint(t1) * (1u << 23) + __float_as_uint(q1));
}

// One 64-column score row (sr) -> numerators in TMEM at t_p.  Adds the sum of the
// unrounded numerators to le.  NPOLY of every 8 column pairs use the polynomial
// exponential.  Numerators are packed and stored to TMEM 32 columns at a time (64 for
// e4m3).
// Keep masks of a 32-key block: bytes >= thr become 0xff (two keys per 16-bit mask half
// below), from the four 64-bit Philox words.
__device__ __forceinline__ void keep_bytes(const uint64_t (&r)[4], uint32_t thr4,
                                           uint32_t (&kb)[8]) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    kb[2 * w] = __vcmpgeu4(static_cast<uint32_t>(r[w]), thr4);
    kb[2 * w + 1] = __vcmpgeu4(static_cast<uint32_t>(r[w] >> 32), thr4);
  }
}

template <bool FP8, int NPOLY, bool DROPOUT = false>
__device__ __forceinline__ void softmax_numerators(const uint32_t (&sr)[4][16], float sl2,
                                                   float neg_m, uint32_t t_p, float &le,
                                                   const uint32_t (*keep)[8] = nullptr) {
  const uint64_t scale2 = ptx::f2_pack(sl2, sl2);
  const uint64_t bias2 = ptx::f2_pack(neg_m, neg_m);
  uint64_t acc_e[2] = {0ull, 0ull};  // packed (0.f, 0.f)
  constexpr int SCOLS = FP8 ? 64 : 32;  // score columns per 16-column TMEM store
#pragma unroll
  for (int q = 0; q < 64 / SCOLS; ++q) {
    uint32_t pk[16];
    float pv[SCOLS];
#pragma unroll
    for (int e = 0; e < SCOLS; e += 2) {
      const int col = q * SCOLS + e;
      const uint64_t xx = ptx::f2_fma(ptx::f2_pack(__uint_as_float(sr[col / 16][col % 16]),
                                                   __uint_as_float(sr[col / 16][col % 16 + 1])),
                                      scale2, bias2);
      float x0, x1;
      ptx::f2_unpack(xx, x0, x1);
      if (((col % 16) / 2) < NPOLY) {
        exp2_poly_pair(x0, x1, pv[e], pv[e + 1]);
      } else {
        pv[e] = ptx::ex2(x0);
        pv[e + 1] = ptx::ex2(x1);
      }
      acc_e[(e / 2) & 1] = ptx::f2_add(acc_e[(e / 2) & 1], ptx::f2_pack(pv[e], pv[e + 1]));
    }
    if (!FP8) {
#pragma unroll
      for (int e = 0; e < SCOLS; e += 2) {
        pk[e / 2] = ptx::pack_bf16x2(pv[e], pv[e + 1]);
        if (DROPOUT) {
          // dropped keys leave the product (not the sum): key byte masks to 16-bit halves
          const uint32_t kb = keep[q][e / 4];
          pk[e / 2] &= ptx::prmt(kb, 0u, (e & 2) ? 0x3322u : 0x1100u);
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < SCOLS; e += 4)
        pk[e / 4] = ptx::pack_e4m3x4(pv[e], pv[e + 1], pv[e + 2], pv[e + 3]);
    }
    ptx::tmem_st16(t_p + q * 16, pk);
  }
  float a0, a1;
  ptx::f2_unpack(ptx::f2_add(acc_e[0], acc_e[1]), a0, a1);
  le += a0 + a1;
}

// Softmax warps: warpgroup x (warps 4x..4x+3) handles Q tile x, one thread per query row
// (TMEM lane).  Every 64-key score tile is loaded whole into registers, masked if it
// crosses the diagonal or the end of the keys, turned into numerators in place, and the
// row statistics are carried from tile to tile.
template <int D, bool CAUSAL, bool OUT_F32, bool FP8, bool VARLEN, bool DROPOUT>
__device__ void softmax_role(const FwdParams &p, uint32_t tmem, const Bars<TileCfg<D, FP8>::NSLOT> &bar,
                             volatile uint32_t *unit_ring, volatile uint32_t *abort_flag,
                             uint8_t *stage) {
  using C = TileCfg<D, FP8>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int x = warp / 4;              // Q tile handled by this warpgroup
  const int wq = warp % 4;             // TMEM lane quarter of this warp
  const int row_in_tile = wq * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t t_o = tmem + lane_base + (x ? C::O_COL1 : C::O_COL0);
  const float NEG_INF = -__int_as_float(0x7f800000);
  uint32_t sph = 0;      // phase bits of s_full(x, b), bit b
  uint32_t pv_base = 0;  // P.V products of this tile in earlier units
  uint32_t unit_it = 0;
  uint32_t taken = 0;

  for (;;) {
    uint32_t u;
    if (!take_unit(bar, unit_ring, taken, abort_flag, ERR_WAIT_SOFTMAX, u) ||
        u >= static_cast<uint32_t>(p.num_units))
      return;
    const Unit w = decode_unit<CAUSAL, VARLEN, C::UNIT>(p, static_cast<int>(u));
    const int nx = x ? w.n1 : w.n0;
    const int row = w.r0 + x * BM + row_in_tile;     // query row of this thread
    const int tile_row0 = w.r0 + x * BM;
    float sl2 = p.scale_log2;
    if (FP8) sl2 *= p.descale_q[w.bh] * p.descale_k[w.bhk];
    // Last admissible key for this row (keys beyond the sequence never count; negative if
    // the row has none).
    const int key_lim = CAUSAL ? min(row + w.off, w.len_k - 1) : w.len_k - 1;
    float m_used = NEG_INF;  // running maximum in use, base-2 scaled domain
    float l = 0.f;           // running sum of the (unrounded, fp32) numerators

    for (int j = 0; j < nx; ++j) {
      const int b = j % C::NBUF;
      bool ok = wait_phase(bar.s_full(x, b), (sph >> b) & 1u, abort_flag, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      sph ^= 1u << b;
      ptx::tc_fence_after();

      const uint32_t t_s = tmem + lane_base + C::s_col(x, b);
      uint32_t sr[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld16(t_s + c * 16, sr[c]);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::reg_fence16(sr[c]);

      const int kv0 = j * BN;
      const bool need_mask =
          (CAUSAL && kv0 + BN - 1 > tile_row0 + w.off) || (kv0 + BN > w.len_k);
      if (need_mask) {
        const int lim = key_lim - kv0;  // column c is admissible iff c <= lim
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c * 16 + e > lim) sr[c][e] = __float_as_uint(NEG_INF);
      }
      // Row maximum: 4 independent chains of three-input maxima.
      float mx[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float m = ptx::max3(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]),
                            __uint_as_float(sr[c][2]));
#pragma unroll
        for (int e = 3; e < 15; e += 2)
          m = ptx::max3(m, __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
        mx[c] = fmaxf(m, __uint_as_float(sr[c][15]));
      }
      const float xmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;

      // Lazy rescale: move m_used only when the new maximum is far above it.
      const bool resc = xmax > m_used + RESCALE_THRESHOLD;
      const float alpha = resc ? ptx::ex2(m_used - xmax) : 1.f;  // 0 on the first tile
      if (__any_sync(0xffffffffu, resc && j > 0)) {
        // The accumulator must be quiescent: wait for P(j-1) V(j-1) of this tile (the
        // products before P(j+1-NBUF) V are covered by the commit that signalled S(j));
        // P(j) V(j) waits for p_full below.
        const uint32_t pn = pv_base + j - 1;  // the previous product of this tile
        ok = wait_phase(bar.pv_done(x, pn & 1u), (pn >> 1) & 1u, abort_flag, ERR_WAIT_SOFTMAX);
        if (!__all_sync(0xffffffffu, ok)) return;
        ptx::tc_fence_after();
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
      if (resc) {
        l *= alpha;
        m_used = xmax;
      }
      const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used;

      // Numerators p = 2^(s*sl2 - m_used), packed for the P V product.  Tiles without
      // masked entries send NPOLY of every 8 column pairs to the FMA-pipe polynomial and
      // the rest to the MUFU unit.
      constexpr int NPOLY = FP8 ? EXP2_POLY_PAIRS_FP8 : EXP2_POLY_PAIRS;
      float le = 0.f;
      const uint32_t t_p = t_s + C::P_OFF;
      if (DROPOUT) {
        // two Philox blocks: keys kv0 .. kv0+31 and kv0+32 .. kv0+63 of this row
        uint32_t keep[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint64_t r[4];
          ptx::philox4x64(static_cast<uint64_t>(kv0 / 32 + h), static_cast<uint64_t>(row),
                          static_cast<uint64_t>(w.bh), 0ull, p.seed, p.offset, r);
          keep_bytes(r, p.drop_thr4, keep[h]);
        }
        softmax_numerators<FP8, 0, true>(sr, sl2, neg_m, t_p, le, keep);
      } else if (NPOLY == 0)   // one copy of the unrolled loop: smaller code, faster
        softmax_numerators<FP8, 0>(sr, sl2, neg_m, t_p, le);
      else if (need_mask)
        softmax_numerators<FP8, 0>(sr, sl2, neg_m, t_p, le);
      else
        softmax_numerators<FP8, NPOLY>(sr, sl2, neg_m, t_p, le);
      // O is normalised by the sum of the unrounded numerators: the bf16 (e4m3) values the
      // tensor core multiplies with V then sum to 1 within one rounding (2^-9 relative for
      // bf16), and the LSE comes from the same sum
      l += le;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar.p_full(x, b));
    }
    pv_base += nx;

    // Epilogue: O = O_acc / l (times the V descale for fp8),
    // LSE = ln 2 * (m_used + log2 l).
    {
      bool ok = wait_phase(bar.o_full(x), unit_it & 1u, abort_flag, ERR_WAIT_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) return;
      ptx::tc_fence_after();
      // a row without admissible keys (causal, more queries than keys) has l = 0: O = 0
      float inv = l > 0.f ? 1.f / l : 0.f;
      if (DROPOUT) inv *= p.keep_scale;
      if (FP8) inv *= p.descale_v[w.bhk];
      // packed varlen output: O [tokens, Hq, d], LSE [Hq, tokens]; the token check keeps
      // the stores inside the tensors whatever the offsets say
      const bool valid = row < w.len_q && (!VARLEN || w.q_tok + row < p.Nq);
      const int hq = w.bh % p.Hq;
      const size_t lrow = VARLEN ? static_cast<size_t>(hq) * p.Nq + w.q_tok + (valid ? row : 0)
                                 : static_cast<size_t>(w.bh) * p.Nq + (valid ? row : 0);
      // O leaves through this warp's staging buffer in shared memory, 32 columns at a time:
      // each thread writes its row's 32 values, then the warp stores whole row segments (8
      // rows of 64 bytes, or 4 rows of 128 bytes, per instruction) instead of 32 scattered
      // 16-byte pieces.  Chunk positions are XOR-swizzled by row, so that neither the
      // row-per-thread writes nor the segment reads meet bank conflicts.
      constexpr int OB = OUT_F32 ? 4 : 2;   // bytes per output element
      constexpr int SEG = 32 * OB;          // bytes of one row's 32 columns
      constexpr int CH = SEG / 16;          // 16-byte chunks per segment
      constexpr int RPI = 32 / CH;          // rows per store instruction
      auto swz = [](int r) { return CH == 8 ? (r & 7) : ((r >> 1) & 3); };
      uint8_t *const st = stage + warp * C::STAGE_WARP_BYTES;
      const int row_w0 = row - lane;        // first row of this warp
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[16], bb[16];
        ptx::tmem_ld16(t_o + c * 32, a);
        ptx::tmem_ld16(t_o + c * 32 + 16, bb);
        ptx::tmem_wait_ld();
        ptx::reg_fence16(a);
        ptx::reg_fence16(bb);
        uint4 v[CH];
        if (OUT_F32) {
#pragma unroll
          for (int q = 0; q < CH; ++q) {
            const uint32_t *s4 = q < 4 ? a + 4 * q : bb + 4 * (q - 4);
            v[q] = make_uint4(__float_as_uint(__uint_as_float(s4[0]) * inv),
                              __float_as_uint(__uint_as_float(s4[1]) * inv),
                              __float_as_uint(__uint_as_float(s4[2]) * inv),
                              __float_as_uint(__uint_as_float(s4[3]) * inv));
          }
        } else {
          uint32_t h[16];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            h[e] = ptx::pack_bf16x2(__uint_as_float(a[2 * e]) * inv, __uint_as_float(a[2 * e + 1]) * inv);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            h[8 + e] = ptx::pack_bf16x2(__uint_as_float(bb[2 * e]) * inv, __uint_as_float(bb[2 * e + 1]) * inv);
#pragma unroll
          for (int q = 0; q < CH; ++q) v[q] = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
#pragma unroll
        for (int q = 0; q < CH; ++q)
          *reinterpret_cast<uint4 *>(st + lane * SEG + (q ^ swz(lane)) * 16) = v[q];
        __syncwarp();
#pragma unroll
        for (int k = 0; k < CH; ++k) {
          const int r = k * RPI + lane / CH, q = lane % CH;
          const uint4 val = *reinterpret_cast<const uint4 *>(st + r * SEG + (q ^ swz(r)) * 16);
          const int rr = row_w0 + r;
          if (rr < w.len_q && (!VARLEN || w.q_tok + rr < p.Nq)) {
            const size_t orr = VARLEN ? static_cast<size_t>(w.q_tok + rr) * p.Hq + hq
                                      : static_cast<size_t>(w.bh) * p.Nq + rr;
            *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.o) + (orr * D + c * 32) * OB +
                                       q * 16) = val;
          }
        }
        __syncwarp();
      }
      if (valid)
        p.lse[lrow] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994530942f : NEG_INF;
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar.o_empty(x));
    }
    ++unit_it;
  }
}

// ---------------------------------------------------------------------------- kernel

template <int D, bool CAUSAL, bool OUT_F32, bool FP8, bool VARLEN, bool DROPOUT = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = TileCfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t smem = (raw + 1023u) & ~1023u;  // 1024-aligned for 128-byte swizzle
  uint8_t *smem_gen = smem_raw + (smem - raw);
  const Bars<C::NSLOT> bar{smem + C::BAR_OFF};
  uint32_t *ctl = reinterpret_cast<uint32_t *>(smem_gen + C::CTL_OFF);
  volatile uint32_t *tmem_slot = ctl;
  volatile uint32_t *abort_flag = ctl + 1;
  volatile uint32_t *unit_ring = ctl + 4;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      ptx::mbar_init(bar.slot_full(s), 1);
      ptx::mbar_init(bar.slot_empty(s), C::NT);   // one arrival per Q tile
    }
    ptx::mbar_init(bar.q_full(), 1);
    ptx::mbar_init(bar.q_empty(), C::NT);
    for (int x = 0; x < 2; ++x) {
      for (int b = 0; b < C::NBUF; ++b) {
        ptx::mbar_init(bar.s_full(x, b), 1);
        ptx::mbar_init(bar.p_full(x, b), BM);
      }
      ptx::mbar_init(bar.pv_done(x, 0), 1);
      ptx::mbar_init(bar.pv_done(x, 1), 1);
      ptx::mbar_init(bar.o_full(x), 1);
      ptx::mbar_init(bar.o_empty(x), BM);
    }
    ptx::mbar_init(bar.drain(0), 1);
    ptx::mbar_init(bar.drain(1), 1);
    for (int s = 0; s < UNIT_RING; ++s) {
      ptx::mbar_init(bar.unit_full(s), 1);
      ptx::mbar_init(bar.unit_empty(s), 5 * C::NT);  // MMA warps + softmax warps
    }
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

  if (warp < 4 * C::NT) {
    softmax_role<D, CAUSAL, OUT_F32, FP8, VARLEN, DROPOUT>(p, tmem, bar, unit_ring, abort_flag,
                                                          smem_gen + C::STAGE_OFF);
  } else if (warp == MMA_WARP || (C::NT == 2 && warp == MMA_WARP + 2)) {
    mma_role<D, CAUSAL, FP8, VARLEN>(p, smem, tmem, bar, warp == MMA_WARP ? 0 : 1, unit_ring,
                                     abort_flag);
    __syncwarp();
  } else if (warp == TMA_WARP) {
    if (lane == 0)
      load_role<D, CAUSAL, FP8, VARLEN>(&tmQ, &tmK, &tmV, p, smem, bar, unit_ring, abort_flag);
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
  // every claim of this CTA is done (its TMA warp has left its loop): count the CTA out;
  // the last one resets the launch's counters
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
  }
}

// Self-test of the bounded wait: one warp waits on the first phase of an mbarrier that
// nothing ever arrives on, with a limit of limit_ns.  The wait runs out, raises
// ERR_WAIT_SELFTEST in the device error word and the kernel returns normally.
__global__ void __launch_bounds__(32, 1) fa_selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_word;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    abort_word = 0u;
    ptx::fence_mbar_init();
  }
  __syncwarp();
  const bool ok = wait_phase_slow(ptx::smem_addr(&bar), 0u, &abort_word, ERR_WAIT_SELFTEST,
                                  limit_ns);
  __syncwarp();
  (void)ok;
}

}  // namespace fa
