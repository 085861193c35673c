// Flash-style sink-augmented GQA prefill on tcgen05 tensor cores.
//
// One CTA owns two 128-row query tiles (A, B) of one (batch, query head) and
// walks the 128-key tiles of the cache the mask admits for them:
//
//   warp 0      TMA producer: K and V tiles of the head's KV group, straight
//               from the cache [B][cap][n_kv][d] (rows past offset+T read as
//               zeros through the tensor map's bounds), NS-deep ring each.
//   warp 1      allocates TMEM and issues every tcgen05.mma from one thread:
//               S_X = Q_X K^T (smem x smem, fp32 in TMEM), then O_X += P_X V
//               with P_X read from TMEM (bf16, aliased over S_X).
//   warps 4-7   softmax for tile A, warps 8-11 for tile B, one query row per
//               thread (TMEM lane = row): load + RoPE the Q row into swizzled
//               smem, then per key tile: mask, running max in log2 units,
//               exp2, P -> TMEM, and at the end O / l -> bf16 out.
//
// The softmax is seeded with the sink logit (m = sink, l = 1), so the extra
// sink column of the MoE-Xtend README ("ATTENTION STACK", sink bias) is
// folded in without ever materialising it, and dropped by construction (it
// adds to l, never to O). The O rescale is lazy: the running max only moves
// when it grows by more than 2^8, which keeps every P <= 256 and the result
// exact up to rounding. Issue order S_A(t) after PV_A(t-1) makes the
// completion of S_A(t) imply that of PV_A(t-1), so a softmax thread may
// rescale O in TMEM as soon as its S is ready.
//
// Key tiles are aligned to tile A's diagonal (key off+i0), so each query
// tile needs a mask only on its diagonal tile, its band edge and the first
// (possibly partial, negative-start) tile; the band layers visit only the
// tiles that intersect [p-W+1, p] -- O(T*W) work.
#pragma once

#include "ptx.cuh"

namespace sa {

struct PrefillParams {
  const __nv_bfloat16* q;
  long long qs0, qs1, qs2;
  __nv_bfloat16* out;
  long long os0, os1, os2;
  float* lse;
  const float* sinks;
  const float* cos_t;
  const float* sin_t;
  int B, T, n_q, n_kv, q_mult;
  long long off;
  int window;
  float scale_log2;
  int rope;
  int n_pairs;
};

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                       // query rows per tile
  static constexpr int BN = 128;                       // keys per tile
  static constexpr int CB = (D % 64 == 0) ? 64 : 32;   // column-block width (elements)
  static constexpr int SWZ = CB * 2;                   // bytes per block row (128 / 64)
  static constexpr int NCB = D / CB;
  static constexpr uint32_t BLOCK_BYTES = 128u * SWZ;  // one column block of a 128-row tile
  static constexpr uint32_t TILE_BYTES = 128u * D * 2;
  static constexpr int NS = (D == 64) ? 4 : (D == 96 ? 3 : 2);  // K and V ring depth
  static constexpr uint32_t LAYOUT = (SWZ == 128) ? 2u : 4u;
  static constexpr uint32_t SBO = 8u * SWZ;            // 8-row core-matrix group stride
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0, S_COL1 = 128;       // S_A, S_B (P aliased in cols [0,64))
  static constexpr int O_COL0 = 256, O_COL1 = 256 + D;
  static constexpr int NUM_THREADS = 384;
  // smem: Q[2] | K[NS] | V[NS] | barriers
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = 2 * TILE_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * TILE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * TILE_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 0, 1);
};

// Barrier slots (8 bytes each) at OFF_BAR.
enum : int {
  BAR_QREADY = 0,  // [2]
  BAR_SFULL = 2,   // [2]
  BAR_PFULL = 4,   // [2]
  BAR_OFINAL = 6,
  BAR_DRAIN = 7,
  BAR_KFULL = 8,   // [NS]
  BAR_KEMPTY = 12, // [NS]
  BAR_VFULL = 16,  // [NS]
  BAR_VEMPTY = 20, // [NS]
  BAR_TMEM_SLOT = 24,
  BAR_ABORT_SLOT = 25,
};

struct TileGeom {
  long long off;
  int T, window;
  int i0;          // first query row of tile A
  long long base;  // first key of key tile 0
  int ntiles;
  __device__ __forceinline__ bool valid(int X) const { return i0 + 128 * X < T; }
  __device__ __forceinline__ long long lo(int X) const {
    const long long p0 = off + i0 + 128 * X;
    return window > 0 ? (p0 - window + 1 > 0 ? p0 - window + 1 : 0) : 0;
  }
  __device__ __forceinline__ long long hi(int X) const {  // exclusive
    const int last = min(T, i0 + 128 * X + 128);
    return off + last;
  }
  __device__ __forceinline__ bool active(int X, int t) const {
    if (t < 0 || t >= ntiles || !valid(X)) return false;
    const long long klo = base + 128LL * t;
    return klo < hi(X) && klo + 128 > lo(X);
  }
  // True when every (row, key) pair of the tile is admitted for all 128 rows.
  __device__ __forceinline__ bool full(int X, int t) const {
    const long long klo = base + 128LL * t;
    const long long p0 = off + i0 + 128 * X;
    if (klo < 0 || klo + 127 > p0) return false;
    if (window > 0 && klo <= p0 + 127 - window) return false;
    return true;
  }
};

__device__ __forceinline__ TileGeom make_geom(const PrefillParams& p, int pair) {
  TileGeom g;
  g.off = p.off;
  g.T = p.T;
  g.window = p.window;
  g.i0 = pair * 256;
  const long long diag = p.off + g.i0;
  const long long loA = g.lo(0);
  const long long nb = (diag - loA + 127) / 128;
  g.base = diag - 128 * nb;
  const long long hi = p.off + min(p.T, g.i0 + 256);
  g.ntiles = (int)((hi - g.base + 127) / 128);
  return g;
}

// MMA issue helpers (one thread). S_X = Q_X K_t^T over d/16 K-steps.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t qbase, uint32_t kbase) {
  using C = PrefillCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t coff = (kk * 16 / C::CB) * C::BLOCK_BYTES + (kk * 16 % C::CB) * 2;
    const uint64_t adesc = smem_desc(qbase + coff, 16, C::SBO, C::LAYOUT);
    const uint64_t bdesc = smem_desc(kbase + coff, 16, C::SBO, C::LAYOUT);
    mma_ss(s_tmem, adesc, bdesc, C::IDESC_QK, kk > 0 ? 1u : 0u);
  }
}
// O_X (+)= P_X V_t over 128/16 K-steps; P_X is bf16 in TMEM (cols [0,64) of S_X).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t vbase,
                                         bool accumulate) {
  using C = PrefillCfg<D>;
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t bdesc = smem_desc(vbase + kk * 16 * C::SWZ, C::BLOCK_BYTES, C::SBO, C::LAYOUT);
    mma_ts(o_tmem, p_tmem + kk * 8, bdesc, C::IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * BAR_TMEM_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * BAR_ABORT_SLOT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = p.n_pairs - 1 - (int)blockIdx.x;  // heaviest query tiles first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / p.q_mult;
  const TileGeom geo = make_geom(p, pair);

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_QREADY + 0), 128);
    mbar_init(bar(BAR_QREADY + 1), 128);
    mbar_init(bar(BAR_SFULL + 0), 1);
    mbar_init(bar(BAR_SFULL + 1), 1);
    mbar_init(bar(BAR_PFULL + 0), 128);
    mbar_init(bar(BAR_PFULL + 1), 128);
    mbar_init(bar(BAR_OFINAL), 1);
    mbar_init(bar(BAR_DRAIN), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_KEMPTY + s), 1);
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // Warpgroup 0: producer (warp 0) and MMA issuer (warp 1); warps 2-3 idle.
    // It gives registers to the two softmax warpgroups: 128*56 + 256*224 =
    // 384*168, the launch allocation.
    regs_dec<56>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ producer
      int issued = 0;
      for (int t = 0; t < geo.ntiles && !*abort_flag; ++t) {
        const int s = t % C::NS;
        const uint32_t ph = (uint32_t)((t / C::NS) & 1);
        const int krow = (int)(geo.base + 128LL * t);
        if (!mbar_wait(bar(BAR_KEMPTY + s), ph ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(bar(BAR_KFULL + s), C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_4d(sbase + C::OFF_K + s * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmK,
                      bar(BAR_KFULL + s), cb * C::CB, g, krow, b);
        issued = t * 2 + 1;
        if (!mbar_wait(bar(BAR_VEMPTY + s), ph ^ 1)) { *abort_flag = 1; break; }
        mbar_arrive_expect_tx(bar(BAR_VFULL + s), C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_4d(sbase + C::OFF_V + s * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmV,
                      bar(BAR_VFULL + s), cb * C::CB, g, krow, b);
        issued = t * 2 + 2;
      }
      if (*abort_flag) {
        // Let every copy still in flight land before the CTA can exit.
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int t = (nk > C::NS ? nk - C::NS : 0); t < nk; ++t)
          mbar_wait(bar(BAR_KFULL + t % C::NS), (uint32_t)((t / C::NS) & 1));
        for (int t = (nv > C::NS ? nv - C::NS : 0); t < nv; ++t)
          mbar_wait(bar(BAR_VFULL + t % C::NS), (uint32_t)((t / C::NS) & 1));
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      bool ok = true;
      if (geo.valid(0) && !mbar_wait(bar(BAR_QREADY + 0), 0)) ok = false;
      if (ok && geo.valid(1) && !mbar_wait(bar(BAR_QREADY + 1), 0)) ok = false;
      tc_fence_after();
      const uint32_t qA = sbase + C::OFF_Q, qB = sbase + C::OFF_Q + C::TILE_BYTES;
      const uint32_t sA = tmem + C::S_COL0, sB = tmem + C::S_COL1;
      const uint32_t oA = tmem + C::O_COL0, oB = tmem + C::O_COL1;
      int nA = 0, nB = 0;  // S tiles issued for A / B (P barrier phases)
      for (int t = 0; t <= geo.ntiles && ok; ++t) {
        const int ks = t % C::NS, vs = (t + C::NS - 1) % C::NS;
        if (t < geo.ntiles) {
          if (!mbar_wait(bar(BAR_KFULL + ks), (uint32_t)((t / C::NS) & 1))) { ok = false; break; }
          tc_fence_after();
        }
        if (t > 0) {
          if (!mbar_wait(bar(BAR_VFULL + vs), (uint32_t)(((t - 1) / C::NS) & 1))) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t kb = sbase + C::OFF_K + ks * C::TILE_BYTES;
        const uint32_t vb = sbase + C::OFF_V + vs * C::TILE_BYTES;
        // tile A: O_A += P_A(t-1) V(t-1), then S_A = Q_A K(t)^T
        if (geo.active(0, t - 1)) {
          if (!mbar_wait(bar(BAR_PFULL + 0), (uint32_t)((nA - 1) & 1))) { ok = false; break; }
          tc_fence_after();
          issue_pv<D>(oA, sA, vb, nA > 1);
        }
        if (t < geo.ntiles && geo.active(0, t)) {
          issue_qk<D>(sA, qA, kb);
          mma_commit(bar(BAR_SFULL + 0));
          ++nA;
        }
        // tile B
        if (geo.active(1, t - 1)) {
          if (!mbar_wait(bar(BAR_PFULL + 1), (uint32_t)((nB - 1) & 1))) { ok = false; break; }
          tc_fence_after();
          issue_pv<D>(oB, sB, vb, nB > 1);
        }
        if (t < geo.ntiles && geo.active(1, t)) {
          issue_qk<D>(sB, qB, kb);
          mma_commit(bar(BAR_SFULL + 1));
          ++nB;
        }
        if (t < geo.ntiles) mma_commit(bar(BAR_KEMPTY + ks));
        if (t > 0) mma_commit(bar(BAR_VEMPTY + vs));
        if (*abort_flag) { ok = false; break; }
      }
      if (ok) {
        mma_commit(bar(BAR_OFINAL));
      } else {
        *abort_flag = 1;
        // Drain the tensor pipe before anything is released.
        mma_commit(bar(BAR_DRAIN));
        mbar_wait(bar(BAR_DRAIN), 0);
        mma_commit(bar(BAR_OFINAL));  // wake the epilogue (its data is discarded)
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    regs_inc<224>();
    const int X = (warp - 4) >> 2;
    const int quarter = warp & 3;               // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;          // row within the query tile
    const int i = geo.i0 + 128 * X + r;         // query row within the call
    const bool row_ok = i < p.T;
    const long long pos = p.off + i;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + (X ? C::S_COL1 : C::S_COL0);
    const uint32_t o_tm = tmem + lane_base + (X ? C::O_COL1 : C::O_COL0);

    if (geo.valid(X)) {
      // Q row -> (RoPE) -> bf16 -> swizzled smem, K-major for the MMA.
      uint8_t* qtile = smem + C::OFF_Q + X * C::TILE_BYTES;
      if (row_ok) {
        const __nv_bfloat16* qrow = p.q + b * p.qs0 + (long long)i * p.qs1 + (long long)h * p.qs2;
        constexpr int HALF = D / 2;
#pragma unroll
        for (int ch = 0; ch < HALF / 8; ++ch) {
          uint4 a = *reinterpret_cast<const uint4*>(qrow + ch * 8);
          uint4 c = *reinterpret_cast<const uint4*>(qrow + HALF + ch * 8);
          if (p.rope) {
            const float4 c0 = *reinterpret_cast<const float4*>(p.cos_t + pos * HALF + ch * 8);
            const float4 c1 = *reinterpret_cast<const float4*>(p.cos_t + pos * HALF + ch * 8 + 4);
            const float4 s0 = *reinterpret_cast<const float4*>(p.sin_t + pos * HALF + ch * 8);
            const float4 s1 = *reinterpret_cast<const float4*>(p.sin_t + pos * HALF + ch * 8 + 4);
            rope_pair2(a.x, c.x, c0.x, c0.y, s0.x, s0.y);
            rope_pair2(a.y, c.y, c0.z, c0.w, s0.z, s0.w);
            rope_pair2(a.z, c.z, c1.x, c1.y, s1.x, s1.y);
            rope_pair2(a.w, c.w, c1.z, c1.w, s1.z, s1.w);
          }
          *reinterpret_cast<uint4*>(qtile + swz_off<C::CB>(r, ch * 8, C::BLOCK_BYTES)) = a;
          *reinterpret_cast<uint4*>(qtile + swz_off<C::CB>(r, HALF + ch * 8, C::BLOCK_BYTES)) = c;
        }
      } else {
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch)
          *reinterpret_cast<uint4*>(qtile + swz_off<C::CB>(r, ch * 8, C::BLOCK_BYTES)) = z;
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(BAR_QREADY + X));

      const float LOG2E = 1.4426950408889634f;
      const float scale = p.scale_log2;
      const float sink2 = p.sinks ? p.sinks[h] * LOG2E : -INFINITY;
      float m = sink2;                              // running max (log2 units)
      float l = (sink2 == -INFINITY) ? 0.f : 1.f;   // running sum, sink included
      int n = 0;
      bool ok = true;
      for (int t = 0; t < geo.ntiles; ++t) {
        if (!geo.active(X, t)) continue;
        if (!mbar_wait(bar(BAR_SFULL + X), (uint32_t)(n & 1))) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(s_tm + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_tm + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(s_tm + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(s_tm + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_wait_ld();
        if (!geo.full(X, t)) {
          // admitted columns c (key klo + c): c >= cmin and c <= cmax
          const long long klo = geo.base + 128LL * t;
          long long lo_k = 0;
          if (p.window > 0 && pos - p.window + 1 > lo_k) lo_k = pos - p.window + 1;
          long long cmin = lo_k - klo, cmax = pos - klo;
          const int cmin_i = (int)(cmin < -1 ? -1 : (cmin > 128 ? 128 : cmin));
          const int cmax_i = (int)(cmax < -1 ? -1 : (cmax > 128 ? 128 : cmax));
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < cmin_i || c > cmax_i) sr[c] = __float_as_uint(-INFINITY);
        }
        // raw row max (scale > 0, so max(s * scale) = scale * max(s))
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          m0 = max3f(m0, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
          m1 = max3f(m1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          m2 = max3f(m2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
          m3 = max3f(m3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
        }
        const float mx = fmaxf(max3f(m0, m1, m2), m3) * scale;
        const float m_new = fmaxf(m, mx);
        const bool need = m_new > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m - m_new) : 1.0f;
          if (n > 0) {
            // O rows stay in TMEM; S_X(t) complete implies PV_X(t-1) complete.
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t rr[32];
              tmem_ld32(o_tm + c0, rr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                float a0 = __uint_as_float(rr[c]), a1 = __uint_as_float(rr[c + 1]);
                mul2(a0, a1, f, f);
                rr[c] = __float_as_uint(a0);
                rr[c + 1] = __float_as_uint(a1);
              }
              tmem_st32(o_tm + c0, rr);
            }
            tmem_wait_st();
          }
          if (need) {
            l *= f;
            m = m_new;
          }
        }
        const float neg = (m == -INFINITY) ? 0.f : -m;
        float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int j = q2 * 64 + 2 * c;
            float x0, x1, x2, x3;
            fma2(x0, x1, __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]), scale, scale, neg, neg);
            fma2(x2, x3, __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]), scale, scale, neg, neg);
            const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
            add2(l0, l1, p0, p1);
            add2(l2, l3, p2, p3);
            pk[c] = pack_bf16(p0, p1);
            pk[c + 1] = pack_bf16(p2, p3);
          }
          tmem_st32(s_tm + q2 * 32, pk);
        }
        l += (l0 + l1) + (l2 + l3);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(BAR_PFULL + X));
        ++n;
        if (*abort_flag) { ok = false; break; }
      }
      // Epilogue: O / l -> bf16.
      if (n > 0 && mbar_wait(bar(BAR_OFINAL), 0) && ok && !*abort_flag) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        __nv_bfloat16* orow = p.out + b * p.os0 + (long long)i * p.os1 + (long long)h * p.os2;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t rr[32];
          tmem_ld32(o_tm + c0, rr);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(rr[c + 0]) * inv_l, __uint_as_float(rr[c + 1]) * inv_l);
              v.y = pack_bf16(__uint_as_float(rr[c + 2]) * inv_l, __uint_as_float(rr[c + 3]) * inv_l);
              v.z = pack_bf16(__uint_as_float(rr[c + 4]) * inv_l, __uint_as_float(rr[c + 5]) * inv_l);
              v.w = pack_bf16(__uint_as_float(rr[c + 6]) * inv_l, __uint_as_float(rr[c + 7]) * inv_l);
              *reinterpret_cast<uint4*>(orow + c0 + c) = v;
            }
          }
        }
        if (row_ok && p.lse) {
          const float LN2 = 0.6931471805599453f;
          p.lse[((long long)b * p.n_q + h) * p.T + i] = (m + __log2f(l)) * LN2;
        }
      } else if (!ok) {
        *abort_flag = 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sa
