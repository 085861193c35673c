// YaRN rotary tables, in-place RoPE of Q/K, and the KV-cache append (with
// optional RoPE of K on the way in). All three are bandwidth-trivial next to
// attention; they are plain coalesced element kernels.
#pragma once

#include "ptx.cuh"

namespace sa {

// x = ((b T + t) H + h) chunks + ch  ->  (b, t, h, ch), with 32-bit
// divisions whenever the index range allows (narrow): a 64-bit division is a
// long software sequence, and three of them per 16 elements made these
// kernels issue-bound.
__device__ __forceinline__ void split_row_chunk(long long x, bool narrow, int chunks, int H, int T, int& b,
                                                int& t, int& h, int& ch) {
  if (narrow) {
    const uint32_t u = (uint32_t)x;
    const uint32_t q1 = u / (uint32_t)chunks, q2 = q1 / (uint32_t)H, q3 = q2 / (uint32_t)T;
    ch = (int)(u - q1 * (uint32_t)chunks);
    h = (int)(q1 - q2 * (uint32_t)H);
    t = (int)(q2 - q3 * (uint32_t)T);
    b = (int)q3;
  } else {
    const long long q1 = x / chunks, q2 = q1 / H, q3 = q2 / T;
    ch = (int)(x - q1 * chunks);
    h = (int)(q1 - q2 * H);
    t = (int)(q2 - q3 * T);
    b = (int)q3;
  }
}

// cos/sin[t][i] = conc * cos/sin(t * inv_freq[i]) per the YaRN + NTK-by-parts
// recipe of the MoE-Xtend README, "ROPE + SCALING": geometric base
// frequencies, extrapolation / interpolation blend through a linear ramp
// between the cutpoints i_beta < i_alpha, concentration 0.1 ln(s) + 1.
// Everything is evaluated in fp64; only the stored result is fp32.
__global__ void yarn_tables_kernel(float* __restrict__ cos_out, float* __restrict__ sin_out,
                                   int max_pos, int half, double theta, double s, double orig_ctx,
                                   double alpha, double beta) {
  const long long n = (long long)max_pos * half;
  const double two_pi = 6.283185307179586476925286766559;
  const double i_beta = half * log(orig_ctx / (beta * two_pi)) / log(theta);
  const double i_alpha = half * log(orig_ctx / (alpha * two_pi)) / log(theta);
  const double conc = 0.1 * log(s) + 1.0;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % half);
    const long long t = idx / half;
    const double freq = pow(theta, (double)i / (double)half);
    const double extrap = 1.0 / freq;
    const double interp = 1.0 / (s * freq);
    double ramp = ((double)i - i_beta) / (i_alpha - i_beta);
    ramp = fmin(fmax(ramp, 0.0), 1.0);
    const double mask = 1.0 - ramp;
    const double inv = interp * (1.0 - mask) + extrap * mask;
    double sn, cs;
    sincos((double)t * inv, &sn, &cs);
    cos_out[idx] = (float)(conc * cs);
    sin_out[idx] = (float)(conc * sn);
  }
}

// Rotate 8 consecutive pairs (x1[c..c+7], x2[c..c+7]) with the table entries
// cos (c0, c1) and sin (s0, s1) already in registers (each result the
// correctly rounded bf16 of the exact rotation; see rope_pair).
__device__ __forceinline__ void rotate8_regs(uint4& a, uint4& b, float4 c0, float4 c1, float4 s0, float4 s1) {
  uint32_t* pa = reinterpret_cast<uint32_t*>(&a);
  uint32_t* pb = reinterpret_cast<uint32_t*>(&b);
  const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) rope_pair2(pa[w], pb[w], cc[2 * w], cc[2 * w + 1], ss[2 * w], ss[2 * w + 1]);
}
// The same with the table entries read from cs[0..7], sn[0..7].
__device__ __forceinline__ void rotate8(uint4& a, uint4& b, const float* __restrict__ cs,
                                       const float* __restrict__ sn) {
  rotate8_regs(a, b, *reinterpret_cast<const float4*>(cs), *reinterpret_cast<const float4*>(cs + 4),
               *reinterpret_cast<const float4*>(sn), *reinterpret_cast<const float4*>(sn + 4));
}

// In-place RoPE of a strided [B][T][H][d] bf16 tensor at positions off + t.
// One thread per (b, t, h, 8-pair chunk).
__global__ void rope_inplace_kernel(__nv_bfloat16* __restrict__ x, long long s0, long long s1,
                                    long long s2, int B, int T, int H, int d, long long off,
                                    const float* __restrict__ cos_t,
                                    const float* __restrict__ sin_t) {
  const int half = d / 2, chunks = half / 8;
  const long long n = (long long)B * T * H * chunks;
  const bool narrow = n <= 0xffffffffLL;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    int b, t, h, ch;
    split_row_chunk(idx, narrow, chunks, H, T, b, t, h, ch);
    __nv_bfloat16* row = x + b * s0 + t * s1 + h * s2;
    uint4 a = *reinterpret_cast<const uint4*>(row + ch * 8);
    uint4 c = *reinterpret_cast<const uint4*>(row + half + ch * 8);
    const long long p = off + t;
    rotate8(a, c, cos_t + p * half + ch * 8, sin_t + p * half + ch * 8);
    *reinterpret_cast<uint4*>(row + ch * 8) = a;
    *reinterpret_cast<uint4*>(row + half + ch * 8) = c;
  }
}

// cache.K[b, off+t, g, :] = rope(k[b, t, g, :]) (or a bit copy when rope == 0),
// cache.V[b, off+t, g, :] = v[b, t, g, :]. One thread per (b, t, g, chunk).
__global__ void kv_append_kernel(__nv_bfloat16* __restrict__ ck, __nv_bfloat16* __restrict__ cv,
                                 int cap, const __nv_bfloat16* __restrict__ k, long long ks0,
                                 long long ks1, long long ks2, const __nv_bfloat16* __restrict__ v,
                                 long long vs0, long long vs1, long long vs2, int B, int T,
                                 int n_kv, int d, long long off, int rope,
                                 const float* __restrict__ cos_t,
                                 const float* __restrict__ sin_t, int ring) {
  const int half = d / 2, chunks = half / 8;
  const long long n = (long long)B * T * n_kv * chunks;
  const bool narrow = n <= 0xffffffffLL;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    int b, t, g, ch;
    split_row_chunk(idx, narrow, chunks, n_kv, T, b, t, g, ch);
    const __nv_bfloat16* krow = k + b * ks0 + t * ks1 + g * ks2;
    const __nv_bfloat16* vrow = v + b * vs0 + t * vs1 + g * vs2;
    uint4 a = *reinterpret_cast<const uint4*>(krow + ch * 8);
    uint4 c = *reinterpret_cast<const uint4*>(krow + half + ch * 8);
    const long long p = off + t;
    if (rope) rotate8(a, c, cos_t + p * half + ch * 8, sin_t + p * half + ch * 8);
    const long long dst = (((long long)b * n_kv + g) * cap + (ring ? p % cap : p)) * d;
    *reinterpret_cast<uint4*>(ck + dst + ch * 8) = a;
    *reinterpret_cast<uint4*>(ck + dst + half + ch * 8) = c;
    *reinterpret_cast<uint4*>(cv + dst + ch * 8) = *reinterpret_cast<const uint4*>(vrow + ch * 8);
    *reinterpret_cast<uint4*>(cv + dst + half + ch * 8) =
        *reinterpret_cast<const uint4*>(vrow + half + ch * 8);
  }
}

// Both this kernel and kv_append_kernel write position p of a ring cache
// (ring != 0) to row p mod cap, else to row p.
// Prefill staging, one launch: the kv_append_kernel work for the call's K/V
// rows, then (stage_q) each query row rotated at its position off + t into
// qo [B][T][n_q][d] (strides os*), from which the attention kernel reads its
// query tiles. One thread per (row, 8-pair chunk); K/V units first. The
// attention kernel, launched behind this one with programmatic stream
// serialization, may be scheduled as soon as every block of this launch has
// started.
__global__ void prefill_stage_kernel(__nv_bfloat16* __restrict__ ck, __nv_bfloat16* __restrict__ cv,
                                     int cap, const __nv_bfloat16* __restrict__ k, long long ks0,
                                     long long ks1, long long ks2, const __nv_bfloat16* __restrict__ v,
                                     long long vs0, long long vs1, long long vs2, int B, int T,
                                     int n_kv, int d, long long off, int rope,
                                     const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                                     const __nv_bfloat16* q, long long qs0, long long qs1,
                                     long long qs2, int n_q, __nv_bfloat16* qo, long long os0,
                                     long long os1, long long os2, int stage_q, int ring) {
  griddep_launch_dependents();
  const int half = d / 2, chunks = half / 8;
  const long long n_kv_units = (long long)B * T * n_kv * chunks;
  const long long n = n_kv_units + (stage_q ? (long long)B * T * n_q * chunks : 0);
  const bool narrow = n <= 0xffffffffLL;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    if (idx < n_kv_units) {
      int b, t, g, ch;
      split_row_chunk(idx, narrow, chunks, n_kv, T, b, t, g, ch);
      const __nv_bfloat16* krow = k + b * ks0 + t * ks1 + g * ks2;
      const __nv_bfloat16* vrow = v + b * vs0 + t * vs1 + g * vs2;
      uint4 a = *reinterpret_cast<const uint4*>(krow + ch * 8);
      uint4 c = *reinterpret_cast<const uint4*>(krow + half + ch * 8);
      const long long p = off + t;
      if (rope) rotate8(a, c, cos_t + p * half + ch * 8, sin_t + p * half + ch * 8);
      const long long dst = (((long long)b * n_kv + g) * cap + (ring ? p % cap : p)) * d;
      *reinterpret_cast<uint4*>(ck + dst + ch * 8) = a;
      *reinterpret_cast<uint4*>(ck + dst + half + ch * 8) = c;
      *reinterpret_cast<uint4*>(cv + dst + ch * 8) = *reinterpret_cast<const uint4*>(vrow + ch * 8);
      *reinterpret_cast<uint4*>(cv + dst + half + ch * 8) =
          *reinterpret_cast<const uint4*>(vrow + half + ch * 8);
    } else {
      const long long iq = idx - n_kv_units;
      int b, t, h, ch;
      split_row_chunk(iq, narrow, chunks, n_q, T, b, t, h, ch);
      const __nv_bfloat16* qrow = q + b * qs0 + t * qs1 + h * qs2;
      __nv_bfloat16* orow = qo + b * os0 + t * os1 + h * os2;
      uint4 a = *reinterpret_cast<const uint4*>(qrow + ch * 8);
      uint4 c = *reinterpret_cast<const uint4*>(qrow + half + ch * 8);
      const long long p = off + t;
      if (rope) rotate8(a, c, cos_t + p * half + ch * 8, sin_t + p * half + ch * 8);
      *reinterpret_cast<uint4*>(orow + ch * 8) = a;
      *reinterpret_cast<uint4*>(orow + half + ch * 8) = c;
    }
  }
}

}  // namespace sa
