// One-token sink-augmented GQA decode, split across SMs.
//
// The work is reading the KV cache once: for each (sequence b, KV head g)
// the rows [lo, off) are cut into S contiguous splits, one CTA each
// (grid n_kv x S x B). Inside a CTA one producer warp streams 128-row K and V
// tiles of head g from the cache with TMA (128-byte swizzled smem, rows past
// `off` read as zeros) through a ring, and eight consumer warps each take
// 16 rows of every tile. A consumer computes S^T = K Q^T for the q_mult <= 8
// query heads of the group with mma.sync m16n8k16 (keys are the M side, the
// heads the N side, so every KV row is read from smem exactly once for the
// whole group), runs the online softmax per head in log2 units, transposes P
// with movmatrix and accumulates O^T = V^T P^T, again on the tensor cores.
//
// The call's new row (position `off`) is rotated, written to the cache and
// attended from registers by the CTA of the last split, so no CTA ever reads
// a cache row written in the same launch.
//
// Partials (m, l, O) of the eight warps are merged in smem; with S > 1 each
// CTA writes its partial to the workspace and the last CTA of (b, g) to
// finish (atomic ticket, no spinning) merges all S of them and folds in the
// sink: M = max(max_s m_s, sink), l = sum_s e^{m_s-M} l_s + e^{sink-M},
// out = sum_s e^{m_s-M} O_s / l.
#pragma once

#include "ptx.cuh"

namespace sa {

struct DecodeParams {
  const __nv_bfloat16* q;
  long long qs0, qs2;
  const __nv_bfloat16* k;
  long long ks0, ks2;
  const __nv_bfloat16* v;
  long long vs0, vs2;
  __nv_bfloat16* ck;
  __nv_bfloat16* cv;
  int cap;
  __nv_bfloat16* out;
  long long os0, os2;
  float* lse;
  const float* sinks;
  const float* cos_t;
  const float* sin_t;
  int B, n_q, n_kv, q_mult;
  long long off;    // position of the new row == cache rows before it
  long long lo;     // first cache position of split 0's first stage
  long long lo_mask;  // first cache position attended (keys before it masked)
  int ring_cap;     // 0: row = position; > 0: ring cache, row = position mod ring_cap
  long long chunk;  // cache rows per split (multiple of 64)
  int S;
  float scale_log2;
  int rope;
  float* ws_o;  // [B][n_kv][S][q_mult][D] (16-byte aligned rows)
  float* ws_m;  // [B][n_kv][S][q_mult]
  float* ws_l;  // [B][n_kv][S][q_mult]
  int* ws_cnt;  // [B][n_kv]
};

template <int D>
struct DecodeCfg {
  static constexpr int NCW = 8;                         // consumer warps
  static constexpr int R = 16 * NCW;                    // rows per stage (16 per consumer warp)
  static constexpr int CB = (D % 64 == 0) ? 64 : 32;
  static constexpr int SWZ = CB * 2;
  static constexpr int NCB = D / CB;
  static constexpr uint32_t BLOCK_BYTES = R * SWZ;       // one column block of a stage
  static constexpr uint32_t STAGE_BYTES = R * D * 2;     // K (or V) of one stage
  static constexpr int NS = (D == 64) ? 3 : 2;
  static constexpr uint32_t XBLOCK = 16 * SWZ;           // column block of the new-row tile
  static constexpr uint32_t XTILE = 16 * D * 2;
  static constexpr int NUM_THREADS = 32 * (NCW + 1);
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = NS * STAGE_BYTES;
  static constexpr uint32_t OFF_XK = 2 * NS * STAGE_BYTES;
  static constexpr uint32_t OFF_XV = OFF_XK + XTILE;
  // [NCW warps][8 m | 8 l | 8*D O] fp32, aliased over the K ring: written only
  // after every consumer warp has finished with the ring
  static constexpr uint32_t OFF_RED = OFF_K;
  static constexpr uint32_t RED_WARP = (16 + 8 * D) * 4;
  static_assert(NCW * RED_WARP <= 2 * NS * STAGE_BYTES, "warp partials must fit in the ring");
  static constexpr uint32_t OFF_BAR = OFF_XV + XTILE;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 8 * (2 * NS) + 16 + 1024;
};

// Warp-level processing of one 16-key sub-tile (rows row0..row0+15 of a tile
// stored as swizzled column blocks of `block_bytes`), keys < n_first and
// keys >= n_valid masked.
template <int D>
__device__ __forceinline__ void decode_subtile(uint32_t kbase, uint32_t vbase, uint32_t block_bytes,
                                               int row0, int n_first, int n_valid,
                                               const uint32_t (&qf)[D / 16][2],
                                               float scale_log2, float (&m)[2], float (&l)[2],
                                               float (&o)[D / 16][4], int lane) {
  using C = DecodeCfg<D>;
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a0, a1, a2, a3;
    const uint32_t addr = kbase + swz_off<C::CB>(row0 + (lane & 15), kk * 16 + 8 * (lane >> 4), block_bytes);
    ldmatrix_x4(addr, a0, a1, a2, a3);
    mma_16816(c, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
  }
  const int key_a = lane >> 2, key_b = key_a + 8;
  float s[4];
  const bool va = key_a >= n_first && key_a < n_valid, vb = key_b >= n_first && key_b < n_valid;
  s[0] = va ? c[0] * scale_log2 : -INFINITY;
  s[1] = va ? c[1] * scale_log2 : -INFINITY;
  s[2] = vb ? c[2] * scale_log2 : -INFINITY;
  s[3] = vb ? c[3] * scale_log2 : -INFINITY;
  float pr[4];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float mx = fmaxf(s[e], s[2 + e]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(m[e], mx);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = ex2(m[e] - m_use);
    pr[e] = ex2(s[e] - m_use);
    pr[2 + e] = ex2(s[2 + e] - m_use);
    l[e] = l[e] * alpha + pr[e] + pr[2 + e];
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      o[md][e] *= alpha;
      o[md][2 + e] *= alpha;
    }
    m[e] = m_new;
  }
  const uint32_t b01 = movmatrix_trans(pack_bf16(pr[0], pr[1]));
  const uint32_t b23 = movmatrix_trans(pack_bf16(pr[2], pr[3]));
#pragma unroll
  for (int md = 0; md < D / 16; ++md) {
    uint32_t a0, a1, a2, a3;
    const int key = (lane & 7) + 8 * (lane >> 4);
    const int col = md * 16 + 8 * ((lane >> 3) & 1);
    ldmatrix_x4_trans(vbase + swz_off<C::CB>(row0 + key, col, block_bytes), a0, a1, a2, a3);
    mma_16816(o[md], a0, a1, a2, a3, b01, b23);
  }
}

template <int D>
__global__ void __launch_bounds__(288, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using C = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) -> uint32_t { return bar0 + 8u * (uint32_t)s; };
  auto empty_bar = [&](int s) -> uint32_t { return bar0 + 8u * (uint32_t)(C::NS + s); };
  volatile int* flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * 2 * C::NS);
  // flag[0]: abort, flag[1]: "this CTA merges the splits"

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;      // KV heads of one split run side by side (same cache rows)
  const int split = blockIdx.y;
  const int b = blockIdx.z;
  const int QM = p.q_mult;
  constexpr int HALF = D / 2;

  const long long r_begin = p.lo + (long long)split * p.chunk;
  long long r_end = r_begin + p.chunk;
  if (r_end > p.off) r_end = p.off;
  const int n_stages = r_end > r_begin ? (int)((r_end - r_begin + C::R - 1) / C::R) : 0;
  const bool last_split = split == p.S - 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::NCW);
    }
    flag[0] = 0;
    flag[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == C::NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_stages > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      for (int it = 0; it < n_stages; ++it) {
        const int s = it % C::NS;
        if (!mbar_wait(empty_bar(s), (uint32_t)(((it / C::NS) & 1) ^ 1))) { flag[0] = 1; break; }
        mbar_arrive_expect_tx(full_bar(s), 2 * C::STAGE_BYTES);
        const long long pos = r_begin + (long long)it * C::R;   // stages never wrap a ring
        const int row = (int)(p.ring_cap > 0 ? pos % p.ring_cap : pos);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_4d(sbase + C::OFF_K + s * C::STAGE_BYTES + cb * C::BLOCK_BYTES, &tmK, full_bar(s),
                      cb * C::CB, row, g, b);
          tma_load_4d(sbase + C::OFF_V + s * C::STAGE_BYTES + cb * C::BLOCK_BYTES, &tmV, full_bar(s),
                      cb * C::CB, row, g, b);
        }
        issued = it + 1;
        if (flag[0]) break;
      }
      if (flag[0]) {
        for (int it = (issued > C::NS ? issued - C::NS : 0); it < issued; ++it)
          mbar_wait_drain(full_bar(it % C::NS), (uint32_t)((it / C::NS) & 1));
      }
    }
    return;  // the producer takes no part in the merge (named barriers below count 32*NCW)
  }

  // ---------------------------------------------------------------- consumers
  // Q fragments (B operand, col-major [d][head]): head n = lane/4 of the group,
  // dims kk*16 + 2*(lane%4) + {0,1} and +8, rotated at position off.
  uint32_t qf[D / 16][2];
  {
    const int n = lane >> 2;
    const bool hv = n < QM;
    const __nv_bfloat16* qrow = p.q + b * p.qs0 + (long long)(g * QM + (hv ? n : 0)) * p.qs2;
    const float* cs = p.cos_t + p.off * HALF;
    const float* sn = p.sin_t + p.off * HALF;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        float y[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = kk * 16 + 8 * hlf + 2 * (lane & 3) + e;
          float x = __bfloat162float(qrow[c]);
          if (p.rope) {
            const int i = c < HALF ? c : c - HALF;
            const float x1 = __bfloat162float(qrow[i]), x2 = __bfloat162float(qrow[i + HALF]);
            uint32_t y1, y2;
            rope_pair(x1, x2, cs[i], sn[i], y1, y2);
            x = __uint_as_float((c < HALF ? y1 : y2) << 16);
          }
          y[e] = hv ? x : 0.f;
        }
        qf[kk][hlf] = pack_bf16(y[0], y[1]);
      }
    }
  }

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[D / 16][4];
#pragma unroll
  for (int md = 0; md < D / 16; ++md) o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;

  // The new row: rotate k, write K/V row `off` of the cache, stage it in smem.
  if (last_split && warp == 0) {
    uint8_t* xk = smem + C::OFF_XK;
    uint8_t* xv = smem + C::OFF_XV;
    const __nv_bfloat16* krow = p.k + b * p.ks0 + (long long)g * p.ks2;
    const __nv_bfloat16* vrow = p.v + b * p.vs0 + (long long)g * p.vs2;
    const long long slot = p.ring_cap > 0 ? p.off % p.ring_cap : p.off;
    __nv_bfloat16* ckrow = p.ck + (((long long)b * p.n_kv + g) * p.cap + slot) * D;
    __nv_bfloat16* cvrow = p.cv + (((long long)b * p.n_kv + g) * p.cap + slot) * D;
    // zero rows 1..15 (and row 0, overwritten below)
    for (int idx = lane; idx < (int)(C::XTILE / 16); idx += 32) {
      reinterpret_cast<uint4*>(xk)[idx] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(xv)[idx] = make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
    for (int c = lane; c < HALF; c += 32) {
      __nv_bfloat16 b1 = krow[c], b2 = krow[c + HALF];
      if (p.rope) {
        uint32_t y1, y2;
        rope_pair(__bfloat162float(b1), __bfloat162float(b2), p.cos_t[p.off * HALF + c],
                  p.sin_t[p.off * HALF + c], y1, y2);
        b1 = __ushort_as_bfloat16((unsigned short)y1);
        b2 = __ushort_as_bfloat16((unsigned short)y2);
      }
      ckrow[c] = b1;
      ckrow[c + HALF] = b2;
      *reinterpret_cast<__nv_bfloat16*>(xk + swz_off<C::CB>(0, c, C::XBLOCK)) = b1;
      *reinterpret_cast<__nv_bfloat16*>(xk + swz_off<C::CB>(0, c + HALF, C::XBLOCK)) = b2;
      const __nv_bfloat16 v1 = vrow[c], v2 = vrow[c + HALF];
      cvrow[c] = v1;
      cvrow[c + HALF] = v2;
      *reinterpret_cast<__nv_bfloat16*>(xv + swz_off<C::CB>(0, c, C::XBLOCK)) = v1;
      *reinterpret_cast<__nv_bfloat16*>(xv + swz_off<C::CB>(0, c + HALF, C::XBLOCK)) = v2;
    }
    __syncwarp();
  }

  for (int it = 0; it < n_stages; ++it) {
    const int s = it % C::NS;
    if (!mbar_wait(full_bar(s), (uint32_t)((it / C::NS) & 1))) { flag[0] = 1; break; }
    const long long row0 = r_begin + (long long)it * C::R + 16 * warp;
    const long long nv = r_end - row0;
    const long long nf = p.lo_mask - row0;
    if (nv > 0 && nf < 16 && !flag[0])
      decode_subtile<D>(sbase + C::OFF_K + s * C::STAGE_BYTES, sbase + C::OFF_V + s * C::STAGE_BYTES,
                        C::BLOCK_BYTES, 16 * warp, nf > 0 ? (int)nf : 0, nv > 16 ? 16 : (int)nv, qf,
                        p.scale_log2, m, l, o, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }
  if (last_split && warp == 0)
    decode_subtile<D>(sbase + C::OFF_XK, sbase + C::OFF_XV, C::XBLOCK, 0, 0, 1, qf, p.scale_log2, m, l,
                      o, lane);

  // ---------------------------------------------------------------- merge the consumer warps
  named_bar_sync(1, 32 * C::NCW);   // every warp is done reading the K/V ring
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 4);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 8);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 16);
  }
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  {
    float* rw = red + warp * (C::RED_WARP / 4);
    const int t = lane & 3;
    if (lane < 4) {
      rw[2 * t] = m[0];
      rw[2 * t + 1] = m[1];
      rw[8 + 2 * t] = l[0];
      rw[8 + 2 * t + 1] = l[1];
    }
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      const int d0 = md * 16 + (lane >> 2);
      rw[16 + (2 * t) * D + d0] = o[md][0];
      rw[16 + (2 * t + 1) * D + d0] = o[md][1];
      rw[16 + (2 * t) * D + d0 + 8] = o[md][2];
      rw[16 + (2 * t + 1) * D + d0 + 8] = o[md][3];
    }
  }
  named_bar_sync(1, 32 * C::NCW);

  const float LOG2E = 1.4426950408889634f, LN2 = 0.6931471805599453f;
  const int tid = threadIdx.x;  // 0 .. 32*NCW-1
  constexpr int NT = 32 * C::NCW;
  const long long slot = ((long long)b * p.n_kv + g) * p.S + split;
  for (int idx = tid; idx < QM * D; idx += NT) {
    const int n = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::NCW; ++w) M = fmaxf(M, red[w * (C::RED_WARP / 4) + n]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < C::NCW; ++w) {
      const float* rw = red + w * (C::RED_WARP / 4);
      const float f = ex2(rw[n] - Mu);
      L += rw[8 + n] * f;
      O += rw[16 + n * D + d] * f;
    }
    const int h = g * QM + n;
    if (p.S == 1) {
      const float sink2 = p.sinks ? p.sinks[h] * LOG2E : -INFINITY;
      const float M2 = fmaxf(M, sink2);
      const float fo = ex2(M - M2);
      const float tot = L * fo + ex2(sink2 - M2);
      p.out[b * p.os0 + (long long)h * p.os2 + d] = __float2bfloat16_rn(O * fo / tot);
      if (d == 0 && p.lse) p.lse[(long long)b * p.n_q + h] = (M2 + __log2f(tot)) * LN2;
    } else {
      p.ws_o[(slot * QM + n) * D + d] = O;
      if (d == 0) {
        p.ws_m[slot * QM + n] = M;
        p.ws_l[slot * QM + n] = L;
      }
    }
  }
  if (p.S == 1) return;

  __threadfence();
  named_bar_sync(1, NT);
  if (tid == 0) {
    const int ticket = atomicAdd(p.ws_cnt + (b * p.n_kv + g), 1);
    flag[1] = (ticket == p.S - 1) ? 1 : 0;
  }
  named_bar_sync(1, NT);
  if (!flag[1]) return;
  __threadfence();

  // Merge the S partials of (b, g). The K/V ring is idle now; reuse it for
  // the per-split weights. Every global read below is batched (independent
  // loads in flight) because this tail runs on one CTA per (b, g) while the
  // rest of the GPU has finished.
  const long long slot0 = ((long long)b * p.n_kv + g) * p.S;
  const int S = p.S;
  float* wsm = reinterpret_cast<float*>(smem);                 // [S][QM] m_s, then e^{m_s - M}
  float* lsm = wsm + (size_t)S * QM;                            // [S][QM] l_s
  float* Msm = lsm + (size_t)S * QM;                            // [QM] M (log2 units)
  float* Lsm = Msm + 8;                                         // [QM] total l
  {
    const float* gm = p.ws_m + slot0 * QM;
    const float* gl = p.ws_l + slot0 * QM;
    const int nml = S * QM;
    int idx = tid;
    for (; idx + 3 * NT < nml; idx += 4 * NT) {
      float a[4], c[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[j] = __ldcg(gm + idx + j * NT);
        c[j] = __ldcg(gl + idx + j * NT);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wsm[idx + j * NT] = a[j];
        lsm[idx + j * NT] = c[j];
      }
    }
    for (; idx < nml; idx += NT) {
      wsm[idx] = __ldcg(gm + idx);
      lsm[idx] = __ldcg(gl + idx);
    }
  }
  named_bar_sync(1, NT);
  {
    // warp w reduces head n = w (QM <= 8 <= NCW): lanes stride over the splits
    const int w = tid >> 5;
    for (int n = w; n < QM; n += C::NCW) {
      const int h = g * QM + n;
      const float sink2 = p.sinks ? p.sinks[h] * LOG2E : -INFINITY;
      float M = sink2;
      for (int s2 = lane; s2 < S; s2 += 32) M = fmaxf(M, wsm[s2 * QM + n]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      float L = 0.f;
      for (int s2 = lane; s2 < S; s2 += 32) {
        const float ms = wsm[s2 * QM + n];
        const float f = (ms == -INFINITY) ? 0.f : ex2(ms - M);
        wsm[s2 * QM + n] = f;
        L += lsm[s2 * QM + n] * f;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
      if (lane == 0) {
        L += ex2(sink2 - M);
        Msm[n] = M;
        Lsm[n] = L;
      }
    }
  }
  named_bar_sync(1, NT);
  {
    // O = sum_s w_s O_s, four consecutive d per thread, eight splits in flight.
    const int nf4 = QM * D / 4;
    const float4* src0 = reinterpret_cast<const float4*>(p.ws_o + slot0 * QM * D);
    for (int idx = tid; idx < nf4; idx += NT) {
      const int n = (idx * 4) / D, d = (idx * 4) % D;
      const float4* src = src0 + idx;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int s2 = 0;
      for (; s2 + 8 <= S; s2 += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __ldcg(src + (size_t)(s2 + j) * nf4);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float w = wsm[(s2 + j) * QM + n];
          acc.x = fmaf(v[j].x, w, acc.x);
          acc.y = fmaf(v[j].y, w, acc.y);
          acc.z = fmaf(v[j].z, w, acc.z);
          acc.w = fmaf(v[j].w, w, acc.w);
        }
      }
      for (; s2 < S; ++s2) {
        const float4 v = __ldcg(src + (size_t)s2 * nf4);
        const float w = wsm[s2 * QM + n];
        acc.x = fmaf(v.x, w, acc.x);
        acc.y = fmaf(v.y, w, acc.y);
        acc.z = fmaf(v.z, w, acc.z);
        acc.w = fmaf(v.w, w, acc.w);
      }
      const int h = g * QM + n;
      const float inv = 1.0f / Lsm[n];
      uint2 packed;
      packed.x = pack_bf16(acc.x * inv, acc.y * inv);
      packed.y = pack_bf16(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(p.out + b * p.os0 + (long long)h * p.os2 + d) = packed;
      if (d == 0 && p.lse) p.lse[(long long)b * p.n_q + h] = (Msm[n] + __log2f(Lsm[n])) * LN2;
    }
  }
  if (tid == 0) p.ws_cnt[b * p.n_kv + g] = 0;
}

}  // namespace sa
