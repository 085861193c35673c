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
// Three launches: a row pass (D and the sink gradient), a key-tile pass (dK,
// dV: one CTA per 64 keys of one KV head, walking the group's heads and the
// query tiles the mask admits) and a query-tile pass (dQ: one CTA per 64
// queries of one head, walking the admitted key tiles). Products run on
// mma.sync m16n8k16 (bf16 operands, fp32 accumulation); P and dS enter their
// products as bf16; outputs are fp32.
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
  float* dvec;           // [B][n_q][T] workspace: D_i
  float* dq;             // [B][T][n_q][d]
  float* dk;             // [B][T][n_kv][d]
  float* dv;             // [B][T][n_kv][d]
  float* dsinks;         // [n_q] or null, zeroed before the launches
  int B, T, n_q, n_kv, q_mult, window;
  float scale;           // sm_scale
  float scale_log2;      // sm_scale * log2(e)
};

// D_i = <dO_i, o_i> per (b, i, h), one warp per row; each row also adds
// -exp(sink_h - lse_i) D_i to dsinks[h].
template <int D>
__global__ void bwd_rows_kernel(const BwdParams p) {
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.B * p.T * p.n_q;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int h = (int)(r % p.n_q);
    const int i = (int)((r / p.n_q) % p.T);
    const int b = (int)(r / ((long long)p.n_q * p.T));
    const __nv_bfloat16* orow = p.o + b * p.os0 + i * p.os1 + h * p.os2;
    const __nv_bfloat16* drow = p.dout + b * p.ds0 + i * p.ds1 + h * p.ds2;
    float acc = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) acc = fmaf(__bfloat162float(orow[c]), __bfloat162float(drow[c]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const long long li = ((long long)b * p.n_q + h) * p.T + i;
      p.dvec[li] = acc;
      if (p.sinks && p.dsinks) atomicAdd(p.dsinks + h, -expf(p.sinks[h] - p.lse[li]) * acc);
    }
  }
}

template <int D>
struct BwdCfg {
  static constexpr int TILE = 64;                 // rows of every tile (4 warps x 16)
  static constexpr int RS = D * 2 + 16;           // padded smem row (bytes): ldmatrix rows hit distinct banks
  static constexpr uint32_t TILE_BYTES = TILE * RS;
  static constexpr uint32_t OFF_A = 0;            // resident tiles -- dK/dV pass: K; dQ pass: Q
  static constexpr uint32_t OFF_B = TILE_BYTES;   //                   V | dO
  // streamed tiles, two buffers -- dK/dV pass: Q, dO; dQ pass: K, V
  static constexpr uint32_t OFF_S = 2 * TILE_BYTES;
  static constexpr uint32_t STREAM_BYTES = 2 * TILE_BYTES;
  // [64] lse and [64] D of the resident (dQ) or streamed (dK/dV, two buffers) query rows
  static constexpr uint32_t OFF_L = OFF_S + 2 * STREAM_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_L + 2 * 512;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Rows [row0, row0 + 64) of a strided [B][T][H][D] bf16 tensor (head and
// batch folded into base) into a padded smem tile by cp.async; rows at or
// past T are zero-filled (no bytes read).
template <int D>
__device__ __forceinline__ void bwd_fetch_tile(uint32_t dst, const __nv_bfloat16* base, long long s1, int row0,
                                               int T) {
  using C = BwdCfg<D>;
  constexpr int CH = D / 8;   // 16-byte chunks per row
  for (int idx = threadIdx.x; idx < C::TILE * CH; idx += blockDim.x) {
    const int r = idx / CH, c = idx % CH;
    const bool in = row0 + r < T;
    const __nv_bfloat16* src = in ? base + (long long)(row0 + r) * s1 + 8 * c : base;
    cp_async16(dst + (uint32_t)(r * C::RS + 16 * c), src, in ? 16u : 0u);
  }
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// lse and D of 64 query rows (contiguous in [B][n_q][T], at any 4-byte
// alignment) into 2 x 64 floats: one element per thread, rows past T zero.
__device__ __forceinline__ void bwd_fetch_rows(uint32_t dst, const float* lse, const float* dvec, int i0, int T) {
  const int t = threadIdx.x;   // 128 threads: lse by 0-63, D by 64-127
  const int r = t & 63;
  const bool in = i0 + r < T;
  const float* src = (t < 64 ? lse : dvec) + (in ? i0 + r : 0);
  cp_async4(dst + (uint32_t)(4 * t), src, in ? 4u : 0u);
}

__device__ __forceinline__ bool bwd_admitted(int i, int j, int T, int window) {
  return i < T && j < T && j <= i && (window <= 0 || j > i - window);
}

// One warp's share of a 64 x 64 block: rows r0..r0+15 of tile X (M side),
// 32 columns c0..c0+31 of tile Y (N side):
//   s = X Y^T and dp = X2 Y2^T over D, returned as 4 n8 accumulator tiles.
template <int D>
__device__ __forceinline__ void bwd_two_products(uint32_t x_base, uint32_t y_base, uint32_t x2_base,
                                                 uint32_t y2_base, int r0, int c0, float (&s)[4][4],
                                                 float (&dp)[4][4], int lane) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t arow = (uint32_t)(r0 + (lane & 15)) * C::RS + (uint32_t)(16 * kk + 8 * (lane >> 4)) * 2;
    uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
    ldmatrix_x4(x_base + arow, a0, a1, a2, a3);
    ldmatrix_x4(x2_base + arow, e0, e1, e2, e3);
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      // B fragments of two n8 tiles from rows (N side) stored [n][k]
      const uint32_t brow = (uint32_t)(c0 + 16 * np + (lane & 7) + 8 * (lane >> 4)) * C::RS +
                            (uint32_t)(16 * kk + 8 * ((lane >> 3) & 1)) * 2;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(y_base + brow, b0, b1, b2, b3);
      mma_16816(s[2 * np], a0, a1, a2, a3, b0, b1);
      mma_16816(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
      ldmatrix_x4(y2_base + brow, b0, b1, b2, b3);
      mma_16816(dp[2 * np], e0, e1, e2, e3, b0, b1);
      mma_16816(dp[2 * np + 1], e0, e1, e2, e3, b2, b3);
    }
  }
}

// acc[D/8][4] += A Z where A (16 x 32) is given as bf16 accumulator pairs of
// 4 n8 tiles (the C -> A fragment identity) and Z is rows k0..k0+31 of a tile
// stored [k][n] (read transposed by ldmatrix).
template <int D>
__device__ __forceinline__ void bwd_accumulate(float (&acc)[D / 8][4], const uint32_t (&ap)[4][2],
                                               uint32_t z_base, int k0, int lane) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kq = 0; kq < 2; ++kq) {
    const uint32_t a0 = ap[2 * kq][0], a1 = ap[2 * kq][1], a2 = ap[2 * kq + 1][0], a3 = ap[2 * kq + 1][1];
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      const uint32_t zaddr = z_base + (uint32_t)(k0 + 16 * kq + (lane & 7) + 8 * ((lane >> 3) & 1)) * C::RS +
                             (uint32_t)(16 * np + 8 * (lane >> 4)) * 2;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(zaddr, b0, b1, b2, b3);
      mma_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
      mma_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}

// dK, dV of keys [j0, j0 + 64) of KV head g, sequence b. K and V stay in
// shared memory; the (head, query tile) pairs stream through two buffers,
// the next pair loading (cp.async) while the current one is computed.
template <int D>
__global__ void __launch_bounds__(128) bwd_dkdv_kernel(const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * C::TILE, g = blockIdx.y, b = blockIdx.z;
  const float LOG2E = 1.4426950408889634f;
  bwd_fetch_tile<D>(sb + C::OFF_A, p.k + b * p.ks0 + (long long)g * p.ks2, p.ks1, j0, p.T);
  bwd_fetch_tile<D>(sb + C::OFF_B, p.v + b * p.vs0 + (long long)g * p.vs2, p.vs1, j0, p.T);
  // query tiles that see some key of this tile: i >= j0, and i < j0 + 63 + W on band layers
  const int qt_lo = j0 / C::TILE;
  int i_end = p.T;
  if (p.window > 0 && j0 + C::TILE - 1 + p.window < i_end) i_end = j0 + C::TILE - 1 + p.window;
  const int nqt = (i_end + C::TILE - 1) / C::TILE - qt_lo;
  const int total = p.q_mult * nqt;
  auto fetch = [&](int idx) {
    const int buf = idx & 1;
    const int h = g * p.q_mult + idx / nqt;
    const int i0 = (qt_lo + idx % nqt) * C::TILE;
    const uint32_t st = sb + C::OFF_S + buf * C::STREAM_BYTES;
    bwd_fetch_tile<D>(st, p.q + b * p.qs0 + (long long)h * p.qs2, p.qs1, i0, p.T);
    bwd_fetch_tile<D>(st + C::TILE_BYTES, p.dout + b * p.ds0 + (long long)h * p.ds2, p.ds1, i0, p.T);
    const long long rb = ((long long)b * p.n_q + h) * p.T;
    bwd_fetch_rows(sb + C::OFF_L + buf * 512, p.lse + rb, p.dvec + rb, i0, p.T);
  };
  fetch(0);
  cp_async_commit();
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
  const int g8 = lane >> 2, t4 = lane & 3;
  for (int idx = 0; idx < total; ++idx) {
    if (idx + 1 < total) {
      fetch(idx + 1);   // into the buffer the previous iteration finished with
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();   // this iteration's tiles (and K, V) are in shared memory
    const int buf = idx & 1;
    const int i0 = (qt_lo + idx % nqt) * C::TILE;
    const uint32_t sq = sb + C::OFF_S + buf * C::STREAM_BYTES, sdo = sq + C::TILE_BYTES;
    const float* sL = reinterpret_cast<const float*>(smem + C::OFF_L + buf * 512);
    const float* sD = sL + 64;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      // S^T (keys x queries) = K Q^T and dP^T = V dO^T for this warp's 16 keys
      float s[4][4], dp[4][4];
      bwd_two_products<D>(sb + C::OFF_A, sq, sb + C::OFF_B, sdo, 16 * warp, 32 * half, s, dp, lane);
      uint32_t pp[4][2], dsp[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float pv[4], dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kr = 16 * warp + g8 + 8 * (e >> 1);
          const int qc = 32 * half + 8 * nt + 2 * t4 + (e & 1);
          const bool ok = bwd_admitted(i0 + qc, j0 + kr, p.T, p.window);
          const float pr = ok ? ex2(s[nt][e] * p.scale_log2 - sL[qc] * LOG2E) : 0.f;
          pv[e] = pr;
          dsv[e] = pr * (dp[nt][e] - sD[qc]);
        }
        pp[nt][0] = pack_bf16(pv[0], pv[1]);
        pp[nt][1] = pack_bf16(pv[2], pv[3]);
        dsp[nt][0] = pack_bf16(dsv[0], dsv[1]);
        dsp[nt][1] = pack_bf16(dsv[2], dsv[3]);
      }
      // dV += P^T dO, dK += dS^T Q over these 32 queries
      bwd_accumulate<D>(dv, pp, sdo, 32 * half, lane);
      bwd_accumulate<D>(dk, dsp, sq, 32 * half, lane);
    }
    __syncthreads();   // every warp is done with this buffer before it is refilled
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int j = j0 + 16 * warp + g8 + 8 * hr;
      if (j >= p.T) continue;
      const long long off = (((long long)b * p.T + j) * p.n_kv + g) * D + 8 * n + 2 * t4;
      *reinterpret_cast<float2*>(p.dk + off) = make_float2(dk[n][2 * hr] * p.scale, dk[n][2 * hr + 1] * p.scale);
      *reinterpret_cast<float2*>(p.dv + off) = make_float2(dv[n][2 * hr], dv[n][2 * hr + 1]);
    }
  }
}

// dQ of queries [i0, i0 + 64) of query head h, sequence b. Q and dO stay in
// shared memory; the admitted K/V tiles stream through two buffers.
template <int D>
__global__ void __launch_bounds__(128) bwd_dq_kernel(const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * C::TILE, h = blockIdx.y, b = blockIdx.z;
  const int g = h / p.q_mult;
  const float LOG2E = 1.4426950408889634f;
  bwd_fetch_tile<D>(sb + C::OFF_A, p.q + b * p.qs0 + (long long)h * p.qs2, p.qs1, i0, p.T);
  bwd_fetch_tile<D>(sb + C::OFF_B, p.dout + b * p.ds0 + (long long)h * p.ds2, p.ds1, i0, p.T);
  const long long rb = ((long long)b * p.n_q + h) * p.T;
  bwd_fetch_rows(sb + C::OFF_L, p.lse + rb, p.dvec + rb, i0, p.T);
  // key tiles these queries see: j <= i, and j > i - W on band layers
  int j_lo = 0;
  if (p.window > 0 && i0 - p.window + 1 > 0) j_lo = i0 - p.window + 1;
  const int kt_lo = j_lo / C::TILE;
  const int total = (min(p.T, i0 + C::TILE) + C::TILE - 1) / C::TILE - kt_lo;
  auto fetch = [&](int idx) {
    const uint32_t st = sb + C::OFF_S + (idx & 1) * C::STREAM_BYTES;
    const int j0 = (kt_lo + idx) * C::TILE;
    bwd_fetch_tile<D>(st, p.k + b * p.ks0 + (long long)g * p.ks2, p.ks1, j0, p.T);
    bwd_fetch_tile<D>(st + C::TILE_BYTES, p.v + b * p.vs0 + (long long)g * p.vs2, p.vs1, j0, p.T);
  };
  fetch(0);
  cp_async_commit();
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;
  const float* sL = reinterpret_cast<const float*>(smem + C::OFF_L);
  const float* sD = sL + 64;
  const int g8 = lane >> 2, t4 = lane & 3;
  for (int idx = 0; idx < total; ++idx) {
    if (idx + 1 < total) {
      fetch(idx + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j0 = (kt_lo + idx) * C::TILE;
    const uint32_t sk = sb + C::OFF_S + (idx & 1) * C::STREAM_BYTES, sv = sk + C::TILE_BYTES;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      // S = Q K^T and dP = dO V^T for this warp's 16 queries and 32 keys
      float s[4][4], dp[4][4];
      bwd_two_products<D>(sb + C::OFF_A, sk, sb + C::OFF_B, sv, 16 * warp, 32 * half, s, dp, lane);
      uint32_t dsp[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qr = 16 * warp + g8 + 8 * (e >> 1);
          const int kc = 32 * half + 8 * nt + 2 * t4 + (e & 1);
          const bool ok = bwd_admitted(i0 + qr, j0 + kc, p.T, p.window);
          const float pr = ok ? ex2(s[nt][e] * p.scale_log2 - sL[qr] * LOG2E) : 0.f;
          dsv[e] = pr * (dp[nt][e] - sD[qr]);
        }
        dsp[nt][0] = pack_bf16(dsv[0], dsv[1]);
        dsp[nt][1] = pack_bf16(dsv[2], dsv[3]);
      }
      // dQ += dS K over these 32 keys
      bwd_accumulate<D>(dq, dsp, sk, 32 * half, lane);
    }
    __syncthreads();
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = i0 + 16 * warp + g8 + 8 * hr;
      if (i >= p.T) continue;
      const long long off = (((long long)b * p.T + i) * p.n_q + h) * D + 8 * n + 2 * t4;
      *reinterpret_cast<float2*>(p.dq + off) = make_float2(dq[n][2 * hr] * p.scale, dq[n][2 * hr + 1] * p.scale);
    }
  }
}

}  // namespace sa
