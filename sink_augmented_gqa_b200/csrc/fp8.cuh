// FP8 (E4M3) KV cache: rows stored as e4m3 codes with one fp32 scale per
// (sequence, position, KV head) row, the format the MoE-Xtend README's
// "ROADMAP" item on quantised long-context KV (dequantisation fused into the
// read) leaves open and this library fixes:
//   amax  = max_d |x_d|           over the bf16 row the bf16 cache would hold
//   scale = fl32(amax / 448)       (one correctly rounded fp32 division)
//   code  = e4m3_rn_satfinite(fl32(x_d / scale)),  a zero row: scale 0, codes 0
// and a reader sees code * scale. Codes live in [B][n_kv][cap][d] bytes,
// scales in [B][n_kv][cap] fp32 (contiguous along positions, so a decode
// stage fetches its 128 scales with one TMA box).
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"

namespace sa {

constexpr float kE4M3Max = 448.0f;

// Two fp32 values to packed e4m3 (lo in the low byte), round to nearest even,
// saturating at +/-448.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two packed e4m3 codes (low byte first) to f16x2 (exact: every e4m3 value
// is an f16 normal or zero).
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t x) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(x));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void mma_16816_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Byte offset of (row, byte column) in a tile stored as column blocks of
// ROWB bytes (block_bytes apart), each block swizzled the way TMA's
// SWIZZLE_{ROWB}B mode writes it: 16-byte chunk index ^= address bits 7.. .
template <int ROWB>
__device__ __forceinline__ uint32_t swz8(int row, int bcol, uint32_t block_bytes) {
  constexpr uint32_t MASK = ROWB / 16 - 1;
  const uint32_t off = (uint32_t)(bcol / ROWB) * block_bytes + (uint32_t)row * ROWB + (uint32_t)(bcol % ROWB);
  return off ^ (((off >> 7) & MASK) << 4);
}

// Address of 32-byte column group grp given the address of group 0 (same row,
// same byte within the group) in a swizzled tile: with ROWB >= 64 the group
// sits in address bits 5.. below the swizzle's source bits, so it is an XOR;
// with 32-byte blocks each group is its own block, block_bytes apart (a
// multiple of 256, which leaves the swizzle unchanged).
template <int ROWB>
__device__ __forceinline__ uint32_t grp_addr(uint32_t a0, int grp, uint32_t block_bytes) {
  return ROWB == 32 ? a0 + (uint32_t)grp * block_bytes : a0 ^ (uint32_t)(32 * grp);
}

// Quantise one row held by a warp, two elements per lane per pass
// (x[i] = elements 2*lane + 64*i, +1; passes with 2*lane + 64*i >= d hold
// zeros and are not stored). Writes codes to dst (device bytes) and returns
// the scale (same value on every lane); codes[i] is the lane's pair of pass i.
template <int NP>
__device__ __forceinline__ float quantize_row_warp(const float (&x)[NP][2], int d, uint8_t* dst,
                                                   int lane, uint16_t (&codes)[NP]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i) amax = fmaxf(amax, fmaxf(fabsf(x[i][0]), fabsf(x[i][1])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = __fdiv_rn(amax, kE4M3Max);
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int c = 2 * lane + 64 * i;
    if (c < d) {
      const uint16_t code = scale == 0.f ? (uint16_t)0
                                         : e4m3x2_from_f32(__fdiv_rn(x[i][0], scale),
                                                           __fdiv_rn(x[i][1], scale));
      *reinterpret_cast<uint16_t*>(dst + c) = code;
      codes[i] = code;
    } else {
      codes[i] = 0;
    }
  }
  return scale;
}

// Append T already-rotated bf16 K/V rows to an FP8 cache at positions
// off + t (ring: row p mod cap). One warp per (b, t, g) row pair.
__global__ void kv_append_fp8_kernel(uint8_t* __restrict__ ck, uint8_t* __restrict__ cv,
                                     float* __restrict__ cks, float* __restrict__ cvs, int cap,
                                     const __nv_bfloat16* __restrict__ k, long long ks0,
                                     long long ks1, long long ks2,
                                     const __nv_bfloat16* __restrict__ v, long long vs0,
                                     long long vs1, long long vs2, int B, int T, int n_kv, int d,
                                     long long off, int ring) {
  const int lane = threadIdx.x & 31;
  const long long n = (long long)B * T * n_kv;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const int g = (int)(r % n_kv);
    const int t = (int)((r / n_kv) % T);
    const int b = (int)(r / ((long long)n_kv * T));
    const __nv_bfloat16* krow = k + b * ks0 + t * ks1 + g * ks2;
    const __nv_bfloat16* vrow = v + b * vs0 + t * vs1 + g * vs2;
    float xk[2][2], xv[2][2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = 2 * lane + 64 * i;
      uint32_t wk = 0, wv = 0;
      if (c < d) {
        wk = *reinterpret_cast<const uint32_t*>(krow + c);
        wv = *reinterpret_cast<const uint32_t*>(vrow + c);
      }
      xk[i][0] = bf16_lo(wk);
      xk[i][1] = bf16_hi(wk);
      xv[i][0] = bf16_lo(wv);
      xv[i][1] = bf16_hi(wv);
    }
    const long long p = off + t;
    const long long row = ((long long)b * n_kv + g) * cap + (ring ? p % cap : p);
    uint16_t codes[2];
    const float sk = quantize_row_warp<2>(xk, d, ck + row * d, lane, codes);
    const float sv = quantize_row_warp<2>(xv, d, cv + row * d, lane, codes);
    if (lane == 0) {
      cks[row] = sk;
      cvs[row] = sv;
    }
  }
}

}  // namespace sa
