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
// HBM-bound: a row is 256 bytes of bf16 in and 128 bytes of codes out.  One kernel does
// the whole job: a cluster of CLUSTER CTAs owns one slice, each CTA an eighth of its rows.
// Pass 1 computes the CTA's amax; the cluster combines the CTAs' values through
// distributed shared memory; pass 2 re-reads the same rows -- from L2, since only a few
// tens of MB stream through the GPU in between -- and writes the codes.  So HBM sees one
// read of the input and one write of the codes.
//
// Thread layout: four threads per row, 8 rows per warp.  The row's 16-byte chunks c =
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

#include "sm100.cuh"

namespace fa {
namespace quant {

constexpr int D = 128;
constexpr int UNIT_ROWS = 8;          // rows per warp-level unit (4 threads per row)
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int CLUSTER = 8;            // CTAs per slice
constexpr float E4M3_MAX = 448.0f;

struct QuantParams {
  const uint16_t *x;                  // bf16 bits [S, N, D]
  const int8_t *signs;                // [D], entry < 0 means -1; nullptr: no rotation
  uint8_t *codes;                     // e4m3 [S, N, D]
  float *descale;                     // [S]
  int rows;                           // N
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

// Load this thread's 32 elements of row `row` (zeros for a row past the slice end) and,
// with ROTATE, apply the signs and the Walsh-Hadamard transform.  zp[k] holds the fp32
// pair at positions (2k, 2k+1).
template <bool ROTATE, bool LAST>
__device__ __forceinline__ void load_transform(const uint16_t *x, long long row, bool valid,
                                               int p, const uint32_t (&m)[16],
                                               uint64_t (&zp)[16]) {
  uint4 raw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    raw[i] = valid ? ld_stream_v4<LAST>(x + row * D + (4 * i + p) * 8) : make_uint4(0, 0, 0, 0);
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
  if (!ROTATE) return;
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

// One slice per cluster: grid = S * CLUSTER CTAs.  CTA c of the cluster takes the units
// (8-row blocks) [c U / CLUSTER, (c+1) U / CLUSTER) of its slice, U = ceil(N / 8), and its
// warps take every WARPS-th unit of that range, so a CTA step covers 64 consecutive rows.
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

  // pass 1: amax of this CTA's rows
  float m = 0.f;
  for (long long u = u0 + warp; u < u1; u += WARPS) {
    const int row0 = static_cast<int>(u * UNIT_ROWS);
    const bool valid = row0 + r < qp.rows;
    uint64_t zp[16];
    load_transform<ROTATE, false>(qp.x, slice * qp.rows + row0 + r, valid, p, m16, zp);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float lo, hi;
      ptx::f2_unpack(zp[k], lo, hi);
      m = ptx::max3(m, fabsf(lo), fabsf(hi));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float c = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) c = fmaxf(c, warp_max[w]);
    cta_max = c;
  }
  // every CTA's cta_max is written before anyone reads it, and read by everyone before
  // any CTA of the cluster may exit
  cluster.sync();
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < CLUSTER; ++c) amax = fmaxf(amax, *cluster.map_shared_rank(&cta_max, c));
  cluster.sync();

  if (crank == 0 && threadIdx.x == 0)
    qp.descale[slice] = amax > 0.f ? amax * qp.norm_over_max : 1.f;
  const float inv = amax > 0.f ? __fdiv_rn(E4M3_MAX, amax) : 0.f;

  // pass 2: the same rows again (now from L2), scaled and rounded to e4m3
  for (long long u = u0 + warp; u < u1; u += WARPS) {
    const int row0 = static_cast<int>(u * UNIT_ROWS);
    const bool valid = row0 + r < qp.rows;
    const long long row = slice * qp.rows + row0 + r;
    uint64_t zp[16];
    load_transform<ROTATE, true>(qp.x, row, valid, p, m16, zp);
    if (valid) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float z[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) ptx::f2_unpack(zp[4 * i + h], z[2 * h], z[2 * h + 1]);
        const uint32_t a = ptx::pack_e4m3x4(z[0] * inv, z[1] * inv, z[2] * inv, z[3] * inv);
        const uint32_t b = ptx::pack_e4m3x4(z[4] * inv, z[5] * inv, z[6] * inv, z[7] * inv);
        st_v2(qp.codes + row * D + 32 * i + 8 * p, a, b);
      }
    }
  }
}

}  // namespace quant
}  // namespace fa
