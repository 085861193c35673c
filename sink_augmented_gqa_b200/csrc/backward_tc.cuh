// Backward pass on tcgen05 tensor cores: the same gradients as backward.cuh,
// from two kernels shaped like the forward prefill kernel:
//
//   MODE 0 (dQ)   rows = 128 queries of one head; streams the admitted key
//                 tiles: S = Q K^T, dP = dO V^T (smem x smem into TMEM),
//                 dS = P (dP - D) as bf16 into TMEM, dQ += dS K (TMEM x smem).
//   MODE 1 (dKdV) rows = 128 keys of one KV head; streams the query tiles
//                 of every head of the group that see them: S^T = K Q^T,
//                 dP^T = V dO^T, P^T and dS^T as bf16 into TMEM, then
//                 dV += P^T dO and dK += dS^T Q.
//
// One CTA per 128-row tile (both passes in one launch, heaviest tiles first),
// 576 threads:
//   warp 0      TMA loads: the two resident 128-row tiles once, then per
//               streamed tile its two BN-row tiles into an NS-deep ring (MODE 1
//               also stages the tile's lse and D values there).
//   warp 1      one thread issues the MMAs and owns the TMEM allocation. S and
//               dP are double-buffered in TMEM: the tensor core computes the
//               next tile's S, dP while this tile's P, dS are formed. P and dS
//               (bf16) get a single buffer of their own where TMEM has room
//               (every case but dK/dV at d = 128): an S / dP buffer is then
//               free as soon as its values are read, and the P / dS warps
//               wait for the previous tile's products only before storing.
//               Otherwise P, dS are written over the S, dP columns they came
//               from, and the issuer waits for tile u - 2's products before
//               tile u reuses that buffer.
//   warps 2-17  P, dS from S, dP: four warps per TMEM lane quarter (warp % 4),
//               each taking a quarter of a tile's columns, one row per thread;
//               tiles wholly inside the admitted region skip the mask; then the
//               fp32 output rows (the warps of a quarter split the columns).
// P_ij = exp2(s_ij scale_log2 - lse_i log2 e) uses the forward's lse (sink
// included), so no running max is needed.
#pragma once

#include "backward.cuh"
#include "ptx.cuh"

namespace sa {

__host__ __device__ constexpr int btc_align32(int x) { return (x + 31) / 32 * 32; }

template <int D, int MODE>
struct BtcCfg {
  static constexpr int BM = 128;                                     // resident rows
  static constexpr int BN = 64;                                      // streamed rows per tile
  static constexpr int CB = (D % 64 == 0) ? 64 : 32;                 // column block (elements)
  static constexpr int SWZ = CB * 2;                                 // bytes per block row
  static constexpr int NCB = D / CB;
  static constexpr uint32_t LAYOUT = (SWZ == 128) ? 2u : 4u;
  static constexpr uint32_t SBO = 8u * SWZ;
  static constexpr uint32_t MBLOCK = (uint32_t)BM * SWZ;
  static constexpr uint32_t M_BYTES = (uint32_t)BM * D * 2;
  static constexpr uint32_t NBLOCK = (uint32_t)BN * SWZ;
  static constexpr uint32_t N_BYTES = (uint32_t)BN * D * 2;
  static constexpr int NS = (D == 128) ? 3 : 4;
  static constexpr uint32_t STAGE_BYTES = 2 * N_BYTES;
  static constexpr uint32_t OFF_R0 = 0;                              // Q (MODE 0) | K (MODE 1)
  static constexpr uint32_t OFF_R1 = M_BYTES;                        // dO | V
  static constexpr uint32_t OFF_ST = 2 * M_BYTES;                    // ring: [K | Q], [V | dO]
  static constexpr uint32_t OFF_ROWV = OFF_ST + NS * STAGE_BYTES;    // MODE 1: [NS][2][BN] fp32
  static constexpr uint32_t OFF_BAR = OFF_ROWV + NS * 2 * BN * 4;
  // at least 120 KB: one CTA per SM, since each allocates all 512 TMEM columns
  static constexpr uint32_t SMEM_BYTES = (OFF_BAR + 256 + 1024) > 120u * 1024 ? (OFF_BAR + 256 + 1024) : 120u * 1024;
  // TMEM columns. S[buf] at S_COL + buf * BN, dP[buf] at DP_COL + buf * BN.
  // SEP: P and dS (bf16 pairs, BN / 2 columns each) have columns of their own
  // after the S / dP buffers, so an S / dP buffer is free again once its
  // values are read; otherwise (dK and dV of d = 128 leave no room) P and dS
  // are written over the start of the S / dP columns they came from.
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = 2 * BN;
  static constexpr bool SEP = 5 * BN + (MODE == 0 ? D : 2 * D) <= 512;
  static constexpr int P_COL = SEP ? 4 * BN : S_COL;                  // MODE 1
  static constexpr int DS_COL = SEP ? 4 * BN + BN / 2 : DP_COL;
  static constexpr int ACC0 = SEP ? 5 * BN : 4 * BN;                  // dQ | dV
  static constexpr int ACC1 = ACC0 + D;                              // MODE 1: dK
  static constexpr int TMEM_COLS = 512;
  static_assert((MODE == 0 ? ACC0 + D : ACC1 + D) <= TMEM_COLS, "TMEM plan exceeds 512 columns");
  static_assert(MBLOCK % 1024 == 0 && NBLOCK % 1024 == 0 && M_BYTES % 1024 == 0, "1 KB aligned tiles");
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
  static constexpr int NSW = 16;                                     // P / dS warps (2..17)
  static constexpr int NPART = NSW / 4;                              // P / dS warps per TMEM lane quarter
  static constexpr int HC = BN / NPART;                              // columns per P / dS warp
  static constexpr int NUM_THREADS = 32 * (2 + NSW);
  static_assert(HC == 16 || HC == 32, "16 or 32 columns per P / dS warp");
  static_assert(NPART % 2 == 0, "dK and dV epilogues take half the warps of a quarter each");
  // the epilogue's 32 x 33 fp32 staging slot per P / dS warp overlays the
  // resident tiles and the ring (below the row values)
  static_assert((uint32_t)NSW * 32 * 33 * 4 <= OFF_ROWV, "epilogue staging overlays tiles and ring");
};

enum : int {
  BB_RFULL = 0,      // resident tiles landed
  BB_FULL = 1,       // [4] ring stage landed
  BB_EMPTY = 5,      // [4] ring stage free (MMA commit)
  BB_SFULL = 9,      // [2] S, dP of a buffer computed
  BB_PFULL = 13,     // count 8 warps: P / dS stored in TMEM
  // 14: unused (the products that read P / dS signal on the stage's EMPTY
  // barrier, which the P / dS warps wait on as well: one commit fewer per tile)
  BB_ACCFULL = 15,   // accumulators final
  BB_DRAIN = 16,
  BB_TMEM_SLOT = 17,
  BB_ABORT_SLOT = 18,
};

// D = sum over K-steps of A (smem, K-major, 128 rows) B (smem, K-major, BN rows)^T
template <int D, int MODE>
__device__ __forceinline__ void btc_issue_s(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc) {
  using C = BtcCfg<D, MODE>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t cb = kk * 16 / C::CB, cin = (kk * 16 % C::CB) * 2;
    mma_ss(d_tmem, adesc + ((cb * C::MBLOCK + cin) >> 4), bdesc + ((cb * C::NBLOCK + cin) >> 4), C::IDESC_S,
           kk > 0 ? 1u : 0u);
  }
}
// acc (+)= A (TMEM bf16, 128 x BN) B (smem [BN][D], MN-major). SEP: A's
// elements sit, as bf16 pairs, at columns [0, BN / 2) of their own buffer;
// otherwise elements [HC h, HC h + HC) sit at columns [HC h, HC h + HC / 2) of
// the S / dP buffer (each P / dS warp writes over the start of the columns it
// read).
template <int D, int MODE>
__device__ __forceinline__ void btc_issue_o(uint32_t acc_tmem, uint32_t a_tmem, uint64_t bdesc, bool accumulate) {
  using C = BtcCfg<D, MODE>;
#pragma unroll
  for (int kk = 0; kk < C::BN / 16; ++kk) {
    const int e = kk * 16;                                        // first element of the K-step
    const uint32_t col = C::SEP ? (uint32_t)(e / 2) : (uint32_t)(C::HC * (e / C::HC) + (e % C::HC) / 2);
    mma_ts(acc_tmem, a_tmem + col, bdesc + ((kk * 16 * C::SWZ) >> 4), C::IDESC_O,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One CTA of either pass: resident row tile `tile` of query head (MODE 0) or
// KV head (MODE 1) `head` of sequence b. tmR0 / tmR1 map the resident tiles'
// tensors, tmS0 / tmS1 the streamed ones (kernel parameters).
template <int D, int MODE>
__device__ __forceinline__ void bwd_tc_cta(const CUtensorMap* tmR0, const CUtensorMap* tmR1,
                                           const CUtensorMap* tmS0, const CUtensorMap* tmS1,
                                           const BwdParams& p, const int tile, const int head, const int b) {
  using C = BtcCfg<D, MODE>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * BB_TMEM_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * BB_ABORT_SLOT);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r0 = tile * C::BM;          // first resident row
  // Streamed tiles. MODE 0: key tiles [t_lo, t_hi) of BN keys seen by
  // queries r0..r0+127. MODE 1: for each head of the group, query tiles
  // [t_lo, t_hi) of BN queries that see keys r0..r0+127.
  int t_lo, t_hi;
  if constexpr (MODE == 0) {
    const int j_lo = p.window > 0 ? max(r0 - p.window + 1, 0) : 0;
    t_lo = j_lo / BN;
    t_hi = (min(p.T, r0 + C::BM) + BN - 1) / BN;
  } else {
    t_lo = r0 / BN;
    int i_end = p.T;
    if (p.window > 0 && r0 + C::BM - 1 + p.window < i_end) i_end = r0 + C::BM - 1 + p.window;
    t_hi = (i_end + BN - 1) / BN;
  }
  const int per = t_hi > t_lo ? t_hi - t_lo : 0;
  const int n_tiles = (MODE == 0) ? per : per * p.q_mult;
  const int g = (MODE == 0) ? head / p.q_mult : head;
  // streamed tile u -> (head of its Q/dO or lse/D rows, first streamed row)
  auto stream_of = [&](int u, int& hh, int& s0) {
    if constexpr (MODE == 0) {
      hh = head;
      s0 = (t_lo + u) * BN;
    } else {
      hh = g * p.q_mult + u / per;
      s0 = (t_lo + u % per) * BN;
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(BB_RFULL), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BB_FULL + s), 1);
      mbar_init(bar(BB_EMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) mbar_init(bar(BB_SFULL + x), 1);
    mbar_init(bar(BB_PFULL), C::NSW);
    mbar_init(bar(BB_ACCFULL), 1);
    mbar_init(bar(BB_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(tmR0);
      tma_prefetch_desc(tmR1);
      tma_prefetch_desc(tmS0);
      tma_prefetch_desc(tmS1);
      mbar_arrive_expect_tx(bar(BB_RFULL), 2 * C::M_BYTES);
      const int rh = (MODE == 0) ? head : g;   // head of the resident tiles
#pragma unroll
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_4d(sbase + C::OFF_R0 + cb * C::MBLOCK, tmR0, bar(BB_RFULL), cb * C::CB, r0, rh, b);
        tma_load_4d(sbase + C::OFF_R1 + cb * C::MBLOCK, tmR1, bar(BB_RFULL), cb * C::CB, r0, rh, b);
      }
    }
    int issued = 0;
    bool ok = true;
    for (int u = 0; u < n_tiles; ++u) {
      const int s = u % C::NS;
      if (u >= C::NS) {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar(BB_EMPTY + s), (uint32_t)(((u / C::NS) - 1) & 1));
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
      }
      if (*abort_flag) { ok = false; break; }
      int hh, s0;
      stream_of(u, hh, s0);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(BB_FULL + s), C::STAGE_BYTES + (MODE == 1 ? 2 * BN * 4 : 0));
        if constexpr (MODE == 1) {
          // lse * log2(e) and D of the tile's BN query rows, beside its tiles
          // (padded workspace rows: 16-byte aligned, valid past T)
          const long long wb = ((long long)b * p.n_q + hh) * p.Tp + s0;
          const uint32_t rv = sbase + C::OFF_ROWV + s * 2 * BN * 4;
          bulk_load(rv, p.lse2 + wb, BN * 4, bar(BB_FULL + s));
          bulk_load(rv + BN * 4, p.dvec + wb, BN * 4, bar(BB_FULL + s));
        }
        const int sh = (MODE == 0) ? g : hh;   // head of the streamed tiles
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_BYTES;
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_4d(st + cb * C::NBLOCK, tmS0, bar(BB_FULL + s), cb * C::CB, s0, sh, b);
          tma_load_4d(st + C::N_BYTES + cb * C::NBLOCK, tmS1, bar(BB_FULL + s), cb * C::CB, s0, sh, b);
        }
      }
      issued = u + 1;
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      for (int u = (issued > C::NS ? issued - C::NS : 0); u < issued; ++u)
        mbar_wait_drain(bar(BB_FULL + u % C::NS), (uint32_t)((u / C::NS) & 1));
    }
    if (lane == 0) mbar_wait_drain(bar(BB_RFULL), 0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(BB_RFULL), 0);
      tc_fence_after();
      const uint64_t a0 = smem_desc(sbase + C::OFF_R0, 16, C::SBO, C::LAYOUT);   // Q | K, K-major
      const uint64_t a1 = smem_desc(sbase + C::OFF_R1, 16, C::SBO, C::LAYOUT);   // dO | V
      auto o_products = [&](int v) {   // the products of tile v that read P / dS
        const int sv = v % C::NS;
        const uint32_t pcol = tmem + C::P_COL + (C::SEP ? 0 : (v & 1) * BN);
        const uint32_t dscol = tmem + C::DS_COL + (C::SEP ? 0 : (v & 1) * BN);
        const uint32_t st = sbase + C::OFF_ST + sv * C::STAGE_BYTES;
        if constexpr (MODE == 0) {
          // dQ += dS K (K of the stage, MN-major)
          btc_issue_o<D, MODE>(tmem + C::ACC0, dscol, smem_desc(st, C::NBLOCK, C::SBO, C::LAYOUT), v > 0);
        } else {
          // dV += P^T dO, dK += dS^T Q
          btc_issue_o<D, MODE>(tmem + C::ACC0, pcol, smem_desc(st + C::N_BYTES, C::NBLOCK, C::SBO, C::LAYOUT),
                               v > 0);
          btc_issue_o<D, MODE>(tmem + C::ACC1, dscol, smem_desc(st, C::NBLOCK, C::SBO, C::LAYOUT), v > 0);
        }
        mma_commit(bar(BB_EMPTY + sv));   // also: tile v's P / dS have been read
      };
      for (int u = 0; u < n_tiles && ok; ++u) {
        const int s = u % C::NS, x = u & 1;
        if (!mbar_wait(bar(BB_FULL + s), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
        // buffer x last served tile u - 2. SEP: its S / dP were read before
        // tile u - 2's P / dS were signalled (waited for below, one tile ago);
        // otherwise wait until the products reading its P / dS completed.
        if (!C::SEP && u >= 2 &&
            !mbar_wait(bar(BB_EMPTY + (u - 2) % C::NS), (uint32_t)(((u - 2) / C::NS) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_BYTES;
        // S = R0 S0^T, dP = R1 S1^T (both K-major)
        btc_issue_s<D, MODE>(tmem + C::S_COL + x * BN, a0, smem_desc(st, 16, C::SBO, C::LAYOUT));
        btc_issue_s<D, MODE>(tmem + C::DP_COL + x * BN, a1, smem_desc(st + C::N_BYTES, 16, C::SBO, C::LAYOUT));
        mma_commit(bar(BB_SFULL + x));
        if (u > 0) {
          if (!mbar_wait(bar(BB_PFULL), (uint32_t)((u - 1) & 1))) { ok = false; break; }
          tc_fence_after();
          o_products(u - 1);
        }
        if (*abort_flag) { ok = false; break; }
      }
      if (ok && n_tiles > 0) {
        if (mbar_wait(bar(BB_PFULL), (uint32_t)((n_tiles - 1) & 1))) {
          tc_fence_after();
          o_products(n_tiles - 1);
          mma_commit(bar(BB_ACCFULL));
        } else {
          ok = false;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(bar(BB_DRAIN));
        mbar_wait_drain(bar(BB_DRAIN), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ dS and the epilogue
    constexpr int HC = C::HC;
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;                    // which HC columns of the tile
    const int rr = quarter * 32 + lane;                  // resident row of this thread
    const int row = r0 + rr;                              // query (MODE 0) or key (MODE 1)
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    float lse2 = 0.f, dval = 0.f;
    if constexpr (MODE == 0) {
      const long long wi = ((long long)b * p.n_q + head) * p.Tp + row;
      if (row < p.Tp) {
        lse2 = p.lse2[wi];
        dval = p.dvec[wi];
      }
    }
    // every wait below is taken warp-uniformly: the TMEM loads and stores
    // that follow are warp-collective
    auto wait_all = [&](uint32_t bb, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bb, parity) ? 1 : 0) != 0;
    };
    bool ok = true;
    for (int u = 0; u < n_tiles && ok; ++u) {
      const int x = u & 1;
      if (!wait_all(bar(BB_SFULL + x), (uint32_t)((u >> 1) & 1))) { ok = false; break; }
      tc_fence_after();
      int hh, s0;
      stream_of(u, hh, s0);
      const int c_base = part * HC;                       // this warp's first column of the tile
      const float* rv = reinterpret_cast<const float*>(smem + C::OFF_ROWV) + (u % C::NS) * 2 * BN;
      if constexpr (MODE == 1) {
        // the producer's lse / D values of this stage: acquire them on the
        // stage's own barrier (its phase cannot move on before this tile's
        // products have run, which wait for these warps)
        if (!wait_all(bar(BB_FULL + u % C::NS), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
      }
      // every (row, column) pair of the tile admitted? (pairs past T are
      // harmless either way: their operand rows are zero or their output
      // rows are not stored)
      bool all_in;
      if constexpr (MODE == 0) {   // rows = queries r0.., columns = keys s0..
        all_in = s0 + BN - 1 <= r0 && (p.window <= 0 || s0 > r0 + C::BM - 1 - p.window);
      } else {                     // rows = keys r0.., columns = queries s0..
        all_in = r0 + C::BM - 1 <= s0 && (p.window <= 0 || r0 > s0 + BN - 1 - p.window);
      }
      uint32_t sv[HC], dv[HC];
      if constexpr (HC == 32) {
        tmem_ld32(tmem + lane_base + C::S_COL + x * BN + c_base, *reinterpret_cast<uint32_t(*)[32]>(sv));
        tmem_ld32(tmem + lane_base + C::DP_COL + x * BN + c_base, *reinterpret_cast<uint32_t(*)[32]>(dv));
      } else {
        tmem_ld16(tmem + lane_base + C::S_COL + x * BN + c_base, sv);
        tmem_ld16(tmem + lane_base + C::DP_COL + x * BN + c_base, dv);
      }
      tmem_wait_ld();
      uint32_t pk[HC / 2], dk[HC / 2];
      float4 lv4 = make_float4(0.f, 0.f, 0.f, 0.f), dv4 = lv4;
#pragma unroll
      for (int c = 0; c < HC; c += 2) {
        float l0, l1, d0, d1;
        if constexpr (MODE == 0) {
          l0 = l1 = lse2;
          d0 = d1 = dval;
        } else {
          if ((c & 3) == 0) {   // the tile's per-column lse / D, four at a time
            lv4 = *reinterpret_cast<const float4*>(rv + c_base + c);
            dv4 = *reinterpret_cast<const float4*>(rv + BN + c_base + c);
          }
          l0 = (c & 3) ? lv4.z : lv4.x;
          l1 = (c & 3) ? lv4.w : lv4.y;
          d0 = (c & 3) ? dv4.z : dv4.x;
          d1 = (c & 3) ? dv4.w : dv4.y;
        }
        float p0, p1;
        fma2(p0, p1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl2, sl2, -l0, -l1);
        // one pair in four on the FMA pipe (the degree-3 exp2 of the
        // forward), the rest on the MUFU unit
        if (((c / 2) & 3) == 0) {
          exp2_fma2(p0, p1);
        } else {
          p0 = ex2(p0);
          p1 = ex2(p1);
        }
        if (!all_in) {
          const int col = s0 + c_base + c;
          if (MODE == 0) {
            if (!bwd_admitted(row, col, p.T, p.window)) p0 = 0.f;
            if (!bwd_admitted(row, col + 1, p.T, p.window)) p1 = 0.f;
          } else {
            if (!bwd_admitted(col, row, p.T, p.window)) p0 = 0.f;
            if (!bwd_admitted(col + 1, row, p.T, p.window)) p1 = 0.f;
          }
        }
        float t0 = __uint_as_float(dv[c]), t1 = __uint_as_float(dv[c + 1]);
        add2(t0, t1, -d0, -d1);
        mul2(t0, t1, p0, p1);
        if constexpr (MODE == 1) pk[c / 2] = pack_bf16(p0, p1);
        dk[c / 2] = pack_bf16(t0, t1);
      }
      uint32_t ps_off;
      if constexpr (C::SEP) {
        // the single P / dS buffer: the previous tile's products must have
        // read it. They signal its stage's EMPTY barrier; that barrier's
        // earlier phase (NS tiles back) is complete here, since the S / dP
        // this warp just read were committed after those products, and its
        // next phase needs this tile's P / dS first.
        if (u >= 1 && !wait_all(bar(BB_EMPTY + (u - 1) % C::NS), (uint32_t)(((u - 1) / C::NS) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        ps_off = (uint32_t)(part * (HC / 2));
      } else {
        // over the start of the S / dP columns this warp read (the other
        // warps of the quarter read and write only their own columns)
        ps_off = (uint32_t)(x * BN + c_base);
      }
      if constexpr (HC == 32) {
        tmem_st16(tmem + lane_base + C::DS_COL + ps_off, dk);
        if constexpr (MODE == 1) tmem_st16(tmem + lane_base + C::P_COL + ps_off, pk);
      } else {
        tmem_st8(tmem + lane_base + C::DS_COL + ps_off, dk);
        if constexpr (MODE == 1) tmem_st8(tmem + lane_base + C::P_COL + ps_off, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BB_PFULL));
      if (*abort_flag) { ok = false; break; }
    }
    // epilogue: the accumulators (zero when no tile was admitted) -> fp32
    // rows. MODE 0: the NPART warps of a quarter take 32-column chunks of dQ
    // in turn; MODE 1: half of them take dV, the other half dK, in turn.
    // Every lane takes part in the TMEM loads; rows past T store nothing.
    const bool have = n_tiles > 0;
    if (ok && have) {
      if (!wait_all(bar(BB_ACCFULL), 0)) ok = false;
      tc_fence_after();
    }
    if (ok) {
      float* out;
      long long rstride;   // elements between consecutive rows of the output
      float mul;
      int acc;
      if constexpr (MODE == 0) {
        out = p.dq + ((long long)b * p.T * p.n_q + head) * D;
        rstride = (long long)p.n_q * D;
        mul = p.scale;
        acc = C::ACC0;
      } else {
        const bool is_dv = part < C::NPART / 2;
        out = (is_dv ? p.dv : p.dk) + ((long long)b * p.T * p.n_kv + head) * D;
        rstride = (long long)p.n_kv * D;
        mul = is_dv ? 1.0f : p.scale;
        acc = is_dv ? C::ACC0 : C::ACC1;
      }
      // Each 32 x 32 chunk (this warp's 32 rows) is transposed through shared
      // memory so that every store instruction writes one row's 128 bytes:
      // a thread-per-row store would scatter 16-byte pieces over 32 rows.
      // The staging slots overlay the resident tiles and the ring, which
      // every product has finished reading once ACCFULL has completed (with
      // no tile there is no such wait: zeros are stored directly).
      float* stg = reinterpret_cast<float*>(smem) + (warp - 2) * (32 * 33);
      const int qrow0 = r0 + quarter * 32;   // first row of this warp's quarter
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        if (MODE == 0 && (c0 / 32) % C::NPART != part) continue;
        if (MODE == 1 && (c0 / 32) % (C::NPART / 2) != part % (C::NPART / 2)) continue;
        if (have) {
          uint32_t a32[32];
          tmem_ld32(tmem + lane_base + acc + c0, a32);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) stg[lane * 33 + c] = __uint_as_float(a32[c]) * mul;
          __syncwarp();
#pragma unroll 4
          for (int r = 0; r < 32; ++r)
            if (qrow0 + r < p.T) out[(long long)(qrow0 + r) * rstride + c0 + lane] = stg[r * 33 + lane];
          __syncwarp();
        } else {
          for (int r = 0; r < 32; ++r)
            if (qrow0 + r < p.T) out[(long long)(qrow0 + r) * rstride + c0 + lane] = 0.f;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Both passes in one launch (they read the same inputs and write disjoint
// outputs), so the tail of one fills with CTAs of the other. Blocks are
// ordered by level k = 0, 1, ...: the n_kv B dK/dV CTAs of key tile k, then
// the n_q B dQ CTAs of query tile tiles - 1 - k; under a causal mask both
// shrink with k, so the heaviest CTAs start first.
template <int D>
__global__ void __launch_bounds__(BtcCfg<D, 0>::NUM_THREADS, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap k1, const __grid_constant__ CUtensorMap v1,
                  const __grid_constant__ CUtensorMap q1, const __grid_constant__ CUtensorMap o1,
                  const __grid_constant__ CUtensorMap q0, const __grid_constant__ CUtensorMap o0,
                  const __grid_constant__ CUtensorMap k0, const __grid_constant__ CUtensorMap v0,
                  const BwdParams p) {
  const int tiles = (p.T + 127) / 128;
  const int nkv = p.n_kv * p.B, nq = p.n_q * p.B;
  const int level = (int)blockIdx.x / (nkv + nq);
  const int r = (int)blockIdx.x % (nkv + nq);
  if (r < nkv)
    bwd_tc_cta<D, 1>(&k1, &v1, &q1, &o1, p, level, r % p.n_kv, r / p.n_kv);
  else
    bwd_tc_cta<D, 0>(&q0, &o0, &k0, &v0, p, tiles - 1 - level, (r - nkv) % p.n_q, (r - nkv) / p.n_q);
}

}  // namespace sa
