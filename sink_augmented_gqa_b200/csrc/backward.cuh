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
// workspace rows, one warp per four rows, which also clears the row's dq
// (the products add into it); each row also adds -exp(sink_h - lse_i) D_i
// to dsinks[h], through a per-block sum in shared memory (dynamic, n_q
// floats) so that global memory sees one atomic per block and head. Rows
// T..Tp-1 get the values of an empty row (D 0, lse +inf).
template <int D>
__global__ void bwd_rows_kernel(const BwdParams p) {
  extern __shared__ float dsink_part[];
  const bool sink = p.sinks && p.dsinks;
  if (sink)
    for (int h = threadIdx.x; h < p.n_q; h += blockDim.x) dsink_part[h] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.B * p.Tp * p.n_q;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  // NR rows per warp and pass, their loads issued before any reduction (rows
  // h, h + 1, ... of one (b, i) are adjacent in o and dO). Row r is (b, i, h)
  // with h fastest; one division per pass (32-bit when the rows allow), the
  // following rows by stepping h.
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
  for (long long r0 = (blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5)) * NR; r0 < rows;
       r0 += warps * NR) {
    int b0, i0, h0;
    split(r0, b0, i0, h0);
    float acc[NR];
    {
      int b = b0, i = i0, h = h0;
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        acc[j] = 0.f;
        if (r0 + j < rows && i < p.T) {
          const __nv_bfloat16* orow = p.o + b * p.os0 + i * p.os1 + h * p.os2;
          const __nv_bfloat16* drow = p.dout + b * p.ds0 + i * p.ds1 + h * p.ds2;
#pragma unroll
          for (int c = lane; c < D; c += 32) acc[j] = fmaf(__bfloat162float(orow[c]), __bfloat162float(drow[c]), acc[j]);
          float* qrow = p.dq + (((long long)b * p.T + i) * p.n_q + h) * D;
#pragma unroll
          for (int c = lane; c < D; c += 32) qrow[c] = 0.f;
        }
        step(b, i, h);
      }
    }
#pragma unroll
    for (int j = 0; j < NR; ++j)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    if (lane < NR && r0 + lane < rows) {
      float a = acc[0];
      int b = b0, i = i0, h = h0;
#pragma unroll
      for (int j = 1; j < NR; ++j) {
        if (lane >= j) {
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
