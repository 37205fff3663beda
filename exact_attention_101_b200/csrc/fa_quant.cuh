// fa_quant.cuh -- per-(batch, head) fp8-e4m3 quantisation of a bf16 [S, N, 128] tensor,
// optionally after the incoherent-processing rotation of the page "FlashAttention-3 (DE)",
// section "Niedrige Praezision (FP8) mit reduziertem Quantisierungsfehler": every row x
// (a query or key vector) is multiplied by the orthogonal matrix R = diag(s) H / sqrt(d),
// with H the d x d Sylvester-Hadamard matrix and s a vector of random signs.  Because
// R R^T = I, (Q R)(K R)^T = Q K^T: the scores are unchanged, while a large entry of x is
// spread over all d coordinates before rounding to 8 bits.
//
// Per slice (one batch and head, N rows):
//   z     = (x * s) H                      (un-normalised Walsh-Hadamard transform, fp32)
//   amax  = max |z| over the slice
//   code  = e4m3_rn_satfinite(z * (448 / amax))          (0 where amax == 0)
//   descale = amax / (448 sqrt(d))                         (1 where amax == 0)
// The normalisation 1/sqrt(d) of R cancels in the codes (z / amax = y / max|y| with
// y = z / sqrt(d)), so it only enters the descale.  Without rotation z = x and the
// descale is amax / 448.
//
// HBM-bound: a row is 256 bytes of bf16 in and 128 bytes of codes out, and the slice
// amax must be known before the first code is written.  A cluster of CTAs owns one slice
// (the amax is combined through distributed shared memory), each CTA a contiguous share of
// its rows:
//  * fa_quant_smem_kernel (slices up to 2048 rows): the CTA copies its whole share (at
//    most 256 rows, 64 KB) into shared memory with bulk asynchronous copies (64-row
//    chunks, one mbarrier each, all in flight at once), computes its amax from there, and
//    after the cluster exchange rounds the same rows from shared memory.  HBM sees one
//    read and one write.
//  * fa_quant_kernel (longer slices): pass 2 re-reads the rows from global memory
//    (partly from L2).  Measured on B200, it beats holding longer slices on chip in
//    clusters of 16 CTAs (which the GPU keeps fewer of in flight).
//// Thread layout: four threads per row, 8 rows per warp.  The row's 16-byte chunks c =
// 0..15 (8 bf16 each) are dealt round-robin: thread p holds chunks 4 i + p, i = 0..3, so
// each load instruction of a warp reads 64 contiguous bytes of each of 8 rows.  Element
// t = 32 i + 8 p + e (e = 0..7) is kept at position q = 8 i + e of the thread.  The
// Walsh-Hadamard strides 1, 2, 4 (bits of e) and 32, 64 (bits of i) stay inside the
// thread; strides 8 and 16 (bits of p) are exchanges with lanes lane^1 and lane^2.  The
// transform is a product of commuting butterflies, so their order does not change the
// exact result.  Values are kept as packed fp32 pairs (q, q+1) for the f32x2 adds.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "fa_fwd_kernel.cuh"  // device error word
#include "sm100.cuh"

namespace fa {
namespace quant {

constexpr int D = 128;
constexpr int UNIT_ROWS = 8;          // rows per warp-level unit (4 threads per row)
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int CLUSTER = 8;            // CTAs per slice of the global-memory kernel
constexpr int MAX_CLUSTER = 8;        // CTAs per slice of the shared-memory kernel
constexpr int ROW_BYTES = D * 2;
constexpr int CHUNK_ROWS = 64;        // rows per bulk copy
constexpr int MAX_SMEM_ROWS = 256;    // rows a CTA holds on chip (64 KB)
constexpr int MAX_CHUNKS = MAX_SMEM_ROWS / CHUNK_ROWS;
constexpr float E4M3_MAX = 448.0f;
constexpr uint32_t ERR_WAIT_QUANT = 1u << 5;

struct QuantParams {
  const uint16_t *x;                  // bf16 bits [S, N, D]
  const int8_t *signs;                // [D], entry < 0 means -1; nullptr: no rotation
  uint8_t *codes;                     // e4m3 [S, N, D]
  float *descale;                     // [S]
  int rows;                           // N
  int cta_rows;                       // shared-memory kernel: rows per CTA (multiple of 8)
  float norm_over_max;                // descale = amax * norm_over_max
};

// 16-byte read-only load that skips L1.  LAST: the second and last read of the data
// (pass 2), with an evict-first L2 policy; otherwise normal L2 priority so that pass 2
// finds the data there.
template <bool LAST>
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  if (LAST) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "l"(pol));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
  }
  return v;
}

__device__ __forceinline__ void st_v2(void *p, uint32_t a, uint32_t b) {
  asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// Sign-flip masks on the raw bf16 pairs: word h of chunk i holds elements t and t + 1
// (t = 32 i + 8 p + 2 h); bit 15 flips t, bit 31 flips t + 1.
__device__ __forceinline__ void load_sign_masks(const int8_t *signs, int p, uint32_t (&m)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int t = 32 * i + 8 * p + 2 * h;
      m[4 * i + h] = (signs[t] < 0 ? 0x8000u : 0u) | (signs[t + 1] < 0 ? 0x80000000u : 0u);
    }
}

// This thread's 32 elements of a row: 16-byte chunks 4 i + p of the row at `src` (global
// memory), zeros for a row past the slice end.
template <bool LAST>
__device__ __forceinline__ void load_raw_global(const uint16_t *src, bool valid, int p,
                                                uint4 (&raw)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    raw[i] = valid ? ld_stream_v4<LAST>(src + (4 * i + p) * 8) : make_uint4(0, 0, 0, 0);
}

// The same from a row held in shared memory at byte address `row_addr`.
__device__ __forceinline__ void load_raw_shared(uint32_t row_addr, bool valid, int p,
                                                uint4 (&raw)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    raw[i] = make_uint4(0, 0, 0, 0);
    if (valid)
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(raw[i].x), "=r"(raw[i].y), "=r"(raw[i].z), "=r"(raw[i].w)
                   : "r"(row_addr + (4 * i + p) * 16));
  }
}

// bf16 -> fp32 and, with ROTATE, the signs and the Walsh-Hadamard transform.  zp[k] holds
// the fp32 pair at positions (2k, 2k+1).
template <bool ROTATE>
__device__ __forceinline__ void transform_raw(const uint4 (&raw)[4], int p,
                                              const uint32_t (&m)[16], uint64_t (&zp)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint32_t v = ROTATE ? (w[h] ^ m[4 * i + h]) : w[h];
      const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xffff0000u);
      // stride 1 of the transform on the two halves of the pair
      zp[4 * i + h] = ROTATE ? ptx::f2_pack(lo + hi, lo - hi) : ptx::f2_pack(lo, hi);
    }
  }
  if constexpr (ROTATE) {
    // in-thread strides 2, 4 (e) and 32, 64 (i): pair-index strides 1, 2, 4, 8
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if ((k & h) == 0) {
          const uint64_t a = zp[k], b = zp[k + h];
          zp[k] = ptx::f2_add(a, b);
          zp[k + h] = ptx::f2_sub(a, b);
        }
    // strides 8 and 16: the lower index of each pair adds, the upper subtracts itself
    // from its partner: z <- other + sgn * z with sgn = +-1 (exact product, one rounding)
#pragma unroll
    for (int bit = 1; bit <= 2; bit <<= 1) {
      const float sg = (p & bit) ? -1.f : 1.f;
      const uint64_t sgn = ptx::f2_pack(sg, sg);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float lo, hi;
        ptx::f2_unpack(zp[k], lo, hi);
        const float olo = __shfl_xor_sync(0xffffffffu, lo, bit);
        const float ohi = __shfl_xor_sync(0xffffffffu, hi, bit);
        zp[k] = ptx::f2_fma(zp[k], sgn, ptx::f2_pack(olo, ohi));
      }
    }
  }
}

__device__ __forceinline__ float abs_max(float m, const uint64_t (&zp)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float lo, hi;
    ptx::f2_unpack(zp[k], lo, hi);
    m = ptx::max3(m, fabsf(lo), fabsf(hi));
  }
  return m;
}

// codes of this thread's 32 elements: element t = 32 i + 8 p + e goes to byte t of the row
__device__ __forceinline__ void store_codes(uint8_t *row_codes, int p, float inv,
                                            const uint64_t (&zp)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float z[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) ptx::f2_unpack(zp[4 * i + h], z[2 * h], z[2 * h + 1]);
    const uint32_t a = ptx::pack_e4m3x4(z[0] * inv, z[1] * inv, z[2] * inv, z[3] * inv);
    const uint32_t b = ptx::pack_e4m3x4(z[4] * inv, z[5] * inv, z[6] * inv, z[7] * inv);
    st_v2(row_codes + 32 * i + 8 * p, a, b);
  }
}

// Block-wide maximum of m (non-negative) into every CTA of the cluster, then the maximum
// over the cluster.  Every thread of every CTA must call it (it holds cluster barriers).
__device__ __forceinline__ float cluster_amax(float m, float *warp_max, float *cta_max) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float c = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) c = fmaxf(c, warp_max[w]);
    *cta_max = c;
  }
  // every CTA's value is written before anyone reads it, and read by everyone before any
  // CTA of the cluster may exit
  cluster.sync();
  float amax = 0.f;
  const int n = static_cast<int>(cluster.num_blocks());
  for (int c = 0; c < n; ++c) amax = fmaxf(amax, *cluster.map_shared_rank(cta_max, c));
  cluster.sync();
  return amax;
}

// Bounded wait for a bulk copy (parity 0: each barrier completes once per launch).
__device__ __forceinline__ bool quant_wait(uint32_t bar) {
  if (ptx::mbar_try_wait(bar, 0)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1; it < WAIT_MAX_ITERS; ++it) {
    if (ptx::mbar_try_wait(bar, 0)) return true;
    if ((it & 255u) == 0 && ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) break;
  }
  atomicOr(&g_fa_error, ERR_WAIT_QUANT);
  return false;
}

// Slices of up to MAX_CLUSTER * MAX_SMEM_ROWS rows: grid = S * cluster CTAs (cluster size
// 1 .. 8, set at launch); CTA c of the cluster holds rows [c * cta_rows, (c+1) * cta_rows) of its
// slice in dynamic shared memory (cta_rows * 256 bytes).  Warp w processes the 8-row units
// w, w + 8, ... of that share, so unit j of a warp lies in chunk j.
template <bool ROTATE>
__global__ void __launch_bounds__(THREADS, 3) fa_quant_smem_kernel(const QuantParams qp) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(128) uint8_t rows_smem[];
  __shared__ __align__(8) uint64_t bars[MAX_CHUNKS];
  __shared__ float warp_max[WARPS];
  __shared__ float cta_max;

  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, p = lane & 3, r = lane >> 2;
  const int cs = static_cast<int>(cluster.num_blocks());
  const long long slice = blockIdx.x / cs;
  const int row_begin = static_cast<int>(cluster.block_rank()) * qp.cta_rows;
  const int nrows = max(0, min(qp.rows - row_begin, qp.cta_rows));
  const int nchunks = (nrows + CHUNK_ROWS - 1) / CHUNK_ROWS;
  const uint16_t *src = qp.x + (slice * qp.rows + row_begin) * D;
  const uint32_t smem_rows = ptx::smem_addr(rows_smem);
  const uint32_t bar0 = ptx::smem_addr(bars);

  if (threadIdx.x == 0) {
    for (int c = 0; c < nchunks; ++c) ptx::mbar_init(bar0 + 8u * c, 1);
    ptx::fence_mbar_init();
    for (int c = 0; c < nchunks; ++c) {
      const int n = min(CHUNK_ROWS, nrows - c * CHUNK_ROWS);
      ptx::mbar_arrive_expect_tx(bar0 + 8u * c, n * ROW_BYTES);
      ptx::bulk_load(smem_rows + c * CHUNK_ROWS * ROW_BYTES, src + c * CHUNK_ROWS * D,
                     n * ROW_BYTES, bar0 + 8u * c);
    }
  }
  uint32_t m16[16] = {};
  if (ROTATE) load_sign_masks(qp.signs, p, m16);
  __syncthreads();

  // pass 1: amax of this CTA's rows, chunk by chunk as the copies land
  float m = 0.f;
  bool ok = true;
  for (int u = warp; u * UNIT_ROWS < nrows; u += WARPS) {
    ok = ok && quant_wait(bar0 + 8u * (u * UNIT_ROWS / CHUNK_ROWS));
    const int row = u * UNIT_ROWS + r;
    uint4 raw[4];
    load_raw_shared(smem_rows + row * ROW_BYTES, ok && row < nrows, p, raw);
    uint64_t zp[16];
    transform_raw<ROTATE>(raw, p, m16, zp);
    m = abs_max(m, zp);
  }
  const float amax = cluster_amax(m, warp_max, &cta_max);
  if (cluster.block_rank() == 0 && threadIdx.x == 0)
    qp.descale[slice] = amax > 0.f ? amax * qp.norm_over_max : 1.f;
  const float inv = amax > 0.f ? __fdiv_rn(E4M3_MAX, amax) : 0.f;

  // pass 2: the same rows from shared memory, scaled and rounded to e4m3
  uint8_t *dst = qp.codes + (slice * qp.rows + row_begin) * D;
  for (int u = warp; u * UNIT_ROWS < nrows; u += WARPS) {
    const int row = u * UNIT_ROWS + r;
    uint4 raw[4];
    load_raw_shared(smem_rows + row * ROW_BYTES, ok && row < nrows, p, raw);
    uint64_t zp[16];
    transform_raw<ROTATE>(raw, p, m16, zp);
    if (ok && row < nrows) store_codes(dst + static_cast<long long>(row) * D, p, inv, zp);
  }
  // a copy that timed out may still be in flight: let it land before the CTA exits
  if (!ok && lane == 0)
    for (int c = 0; c < nchunks; ++c) quant_wait(bar0 + 8u * c);
}

// Longer slices: grid = S * CLUSTER CTAs, one slice per cluster.  CTA c of the cluster
// takes the units (8-row blocks) [c U / CLUSTER, (c+1) U / CLUSTER) of its slice,
// U = ceil(N / 8), and its warps take every WARPS-th unit of that range, so a CTA step
// covers 64 consecutive rows.  Pass 2 re-reads the rows from global memory.
template <bool ROTATE>
__global__ void __cluster_dims__(CLUSTER, 1, 1) __launch_bounds__(THREADS, 3)
    fa_quant_kernel(const QuantParams qp) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float warp_max[WARPS];
  __shared__ float cta_max;

  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, p = lane & 3, r = lane >> 2;
  const int crank = static_cast<int>(cluster.block_rank());
  const long long slice = blockIdx.x / CLUSTER;
  const long long per_slice = (qp.rows + UNIT_ROWS - 1) / UNIT_ROWS;
  const long long u0 = per_slice * crank / CLUSTER, u1 = per_slice * (crank + 1) / CLUSTER;
  uint32_t m16[16] = {};
  if (ROTATE) load_sign_masks(qp.signs, p, m16);

  float m = 0.f;
  for (long long u = u0 + warp; u < u1; u += WARPS) {
    const long long row = u * UNIT_ROWS + r;
    uint4 raw[4];
    load_raw_global<false>(qp.x + (slice * qp.rows + row) * D, row < qp.rows, p, raw);
    uint64_t zp[16];
    transform_raw<ROTATE>(raw, p, m16, zp);
    m = abs_max(m, zp);
  }
  const float amax = cluster_amax(m, warp_max, &cta_max);
  if (crank == 0 && threadIdx.x == 0)
    qp.descale[slice] = amax > 0.f ? amax * qp.norm_over_max : 1.f;
  const float inv = amax > 0.f ? __fdiv_rn(E4M3_MAX, amax) : 0.f;

  for (long long u = u0 + warp; u < u1; u += WARPS) {
    const long long row = u * UNIT_ROWS + r;
    const long long g = slice * qp.rows + row;
    uint4 raw[4];
    load_raw_global<true>(qp.x + g * D, row < qp.rows, p, raw);
    uint64_t zp[16];
    transform_raw<ROTATE>(raw, p, m16, zp);
    if (row < qp.rows) store_codes(qp.codes + g * D, p, inv, zp);
  }
}

}  // namespace quant
}  // namespace fa
