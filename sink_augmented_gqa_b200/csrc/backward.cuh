// Backward pass of sink-augmented GQA attention (training the sinks end to
// end; GPT-OSS-Lite README, "Architecture": learned attention sinks), for a
// sequence attending to itself (no cache prefix), on the rotated q and k:
//
//   P_ij = exp(s_ij - lse_i), s_ij = sm_scale <q_i, k_j> on admitted pairs,
//   lse_i the forward's log-sum-exp including the sink column;
//   D_i = <dO_i, o_i>;  dP_ij = <dO_i, v_j>;  dS_ij = P_ij (dP_ij - D_i);
//   dq_i = sm_scale sum_j dS_ij k_j;   dk_j = sm_scale sum dS_ij q_i;
//   dv_j = sum P_ij dO_i  (dk, dv summed over the heads of the KV group);
//   dsink_h = -sum_{b,i} exp(sink_h - lse_i) D_i  (the sink carries no value).
//
// Two launches: the row pass below (D, the sink gradient, and dq cleared),
// then the products of backward_tc.cuh on the tcgen05 tensor cores (bf16
// operands, fp32 accumulation in TMEM; P and dS enter their products as
// bf16), which accumulate dq with reductions; outputs are fp32.
#pragma once

#include "ptx.cuh"

namespace sa {

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  long long qs0, qs1, qs2, ks0, ks1, ks2, vs0, vs1, vs2, os0, os1, os2, ds0, ds1, ds2;
  const float* lse;      // [B][n_q][T], natural log
  const float* sinks;    // [n_q] or null
  float* dvec;           // [B][n_q][Tp] workspace: D_i (0 for rows past T)
  float* lse2;           // [B][n_q][Tp] workspace: lse_i * log2(e) (+inf for rows past T)
  int Tp;                // T rounded up to a multiple of 384 (whole streamed tiles of 64, 96 or 128 rows)
  float* dq;             // [B][T][n_q][d]
  float* dk;             // [B][T][n_kv][d]
  float* dv;             // [B][T][n_kv][d]
  float* dsinks;         // [n_q] or null, zeroed before the launches
  int B, T, n_q, n_kv, q_mult, window;
  float scale;           // sm_scale
  float scale_log2;      // sm_scale * log2(e)
};

// D_i = <dO_i, o_i> and lse_i log2(e) per (b, i, h) into the padded
// workspace rows; the row's dq is cleared on the way (the products add into
// it). Half a warp per row, 16-byte pieces (d / 8 lanes read o and dO, all 16
// clear dq), four rows per half-warp and pass with every load issued before
// any reduction. Each row also adds -exp(sink_h - lse_i) D_i to dsinks[h],
// through a per-block sum in shared memory (dynamic, n_q floats) so that
// global memory sees one atomic per block and head. Rows T..Tp-1 get the
// values of an empty row (D 0, lse +inf).
template <int D>
__global__ void bwd_rows_kernel(const BwdParams p) {
  extern __shared__ float dsink_part[];
  const bool sink = p.sinks && p.dsinks;
  if (sink)
    for (int h = threadIdx.x; h < p.n_q; h += blockDim.x) dsink_part[h] = 0.f;
  __syncthreads();
  constexpr int CH = D / 8;   // 16-byte pieces of a bf16 row (8, 12 or 16)
  static_assert(CH <= 16, "a row fits half a warp");
  const int sub = threadIdx.x & 15;
  const long long rows = (long long)p.B * p.Tp * p.n_q;
  const long long groups = (long long)gridDim.x * (blockDim.x >> 4);
  // Row r is (b, i, h) with h fastest (rows h, h + 1, ... of one (b, i) are
  // adjacent in o and dO); one division per pass (32-bit when the rows
  // allow), the following rows by stepping h.
  constexpr int NR = 4;
  auto split = [&](long long r, int& b, int& i, int& h) {
    if (rows <= 0xffffffffLL) {
      const uint32_t ru = (uint32_t)r, t = ru / (uint32_t)p.n_q;
      h = (int)(ru - t * (uint32_t)p.n_q);
      i = (int)(t % (uint32_t)p.Tp);
      b = (int)(t / (uint32_t)p.Tp);
    } else {
      const long long t = r / p.n_q;
      h = (int)(r - t * p.n_q);
      i = (int)(t % p.Tp);
      b = (int)(t / p.Tp);
    }
  };
  auto step = [&](int& b, int& i, int& h) {
    if (++h == p.n_q) {
      h = 0;
      if (++i == p.Tp) {
        i = 0;
        ++b;
      }
    }
  };
  for (long long r0 = (blockIdx.x * (long long)(blockDim.x >> 4) + (threadIdx.x >> 4)) * NR; r0 < rows;
       r0 += groups * NR) {
    int b0, i0, h0;
    split(r0, b0, i0, h0);
    uint4 ov[NR], dv[NR];
    {
      int b = b0, i = i0, h = h0;
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        ov[j] = dv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (r0 + j < rows && i < p.T) {
          if (sub < CH) {
            ov[j] = *reinterpret_cast<const uint4*>(p.o + b * p.os0 + i * p.os1 + h * p.os2 + sub * 8);
            dv[j] = *reinterpret_cast<const uint4*>(p.dout + b * p.ds0 + i * p.ds1 + h * p.ds2 + sub * 8);
          }
          float4* qrow = reinterpret_cast<float4*>(p.dq + (((long long)b * p.T + i) * p.n_q + h) * D);
#pragma unroll
          for (int c = sub; c < D / 4; c += 16) qrow[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        step(b, i, h);
      }
    }
    float acc[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      const uint32_t* o2 = reinterpret_cast<const uint32_t*>(&ov[j]);
      const uint32_t* d2 = reinterpret_cast<const uint32_t*>(&dv[j]);
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a = fmaf(bf16_lo(o2[e]), bf16_lo(d2[e]), a);
        a = fmaf(bf16_hi(o2[e]), bf16_hi(d2[e]), a);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      acc[j] = a;
    }
    if (sub < NR && r0 + sub < rows) {
      float a = acc[0];
      int b = b0, i = i0, h = h0;
#pragma unroll
      for (int j = 1; j < NR; ++j) {
        if (sub >= j) {
          a = acc[j];
          step(b, i, h);
        }
      }
      const long long wi = ((long long)b * p.n_q + h) * p.Tp + i;
      if (i >= p.T) {
        p.dvec[wi] = 0.f;
        p.lse2[wi] = INFINITY;
      } else {
        const long long li = ((long long)b * p.n_q + h) * p.T + i;
        p.dvec[wi] = a;
        p.lse2[wi] = p.lse[li] * 1.4426950408889634f;
        if (sink) atomicAdd(dsink_part + h, -expf(p.sinks[h] - p.lse[li]) * a);
      }
    }
  }
  if (sink) {
    __syncthreads();
    for (int h = threadIdx.x; h < p.n_q; h += blockDim.x) atomicAdd(p.dsinks + h, dsink_part[h]);
  }
}

__device__ __forceinline__ bool bwd_admitted(int i, int j, int T, int window) {
  return i < T && j < T && j <= i && (window <= 0 || j > i - window);
}

}  // namespace sa
