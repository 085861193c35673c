// Backward pass on tcgen05 tensor cores: every gradient of backward.cuh
// (dQ, dK, dV) from one launch whose CTAs each keep 128 keys of one KV head
// resident and stream the query tiles of every head of the group that see
// them:
//
//   S^T  = K Q^T,  dP^T = V dO^T          smem x smem into TMEM (keys = TMEM lanes)
//   P^T  = exp2(S^T scale log2 e - lse log2 e),  dS^T = P^T (dP^T - D)
//          formed by 16 warps, one key row per thread, and written as bf16
//          to shared memory in the layouts the next products read
//   dV  += P^T dO,  dK += dS^T Q          accumulated in TMEM over the CTA's tiles
//   dQ^T = K^T dS^T                        per tile, into TMEM; the same warps
//          stage it as [query][d] fp32 rows in the ring slot its tile's Q and
//          dO have just left (the same byte count), and the TMA thread adds
//          the rows to dq with a tensor reduce-add before refilling the slot
//
// Five products per (key, query) pair: S and dP are formed once for all
// three gradients. BN, the query rows of a streamed tile, is what TMEM holds
// next to the accumulators: S^T, dP^T and dQ^T (BN columns each), dV, dK (D
// each): 3 BN + 2 D <= 512 gives BN = 128 at d = 64, 96 at d = 96, 64 at
// d = 128. dQ^T's products have M = 128 rows of d; at d < 128 the rows past d
// read the start of the V tile (stored right after K) and are never read
// back.
//
// 576 threads per CTA, one CTA per SM (each holds all 512 TMEM columns):
//   warp 0      TMA: K and V once; per streamed tile its Q and dO tiles and
//               the tile's lse log2 e and D values (bulk copies) into an
//               NS-deep ring; each slot is refilled once the dQ^T rows staged
//               in it have been read by their reduce-add.
//   warp 1      one thread issues the MMAs and owns the TMEM allocation. It
//               issues tile u's S^T, dP^T as soon as the warps have read tile
//               u - 1's, then tile u - 1's dV, dK and dQ^T products once its
//               P^T, dS^T are in shared memory: the tensor cores form the
//               next scores while the warps work on the current tile.
//   warps 2-17  P^T, dS^T from S^T, dP^T (four warps per TMEM lane quarter,
//               each a quarter of the tile's columns); then, once the previous
//               tile's products are done, that tile's dQ^T into the staging
//               rows (the warps of the lane quarters that hold d rows), and
//               this tile's P^T, dS^T into shared memory; at the end dV, dK
//               (fp32 rows).
// Adding dq's partial sums is what bounds this kernel: each 128-key tile adds
// a BN x d fp32 block per query tile, and the reduce-adds move about 8-9
// bytes per SM cycle (the ring slot they read is refilled only afterwards).
// dq must be zero before the launch (the row pass clears it). The order in
// which the key tiles' contributions reach a dq element varies, so dq can
// differ in the last bits between calls; dk and dv do not.
#pragma once

#include "backward.cuh"
#include "ptx.cuh"

namespace sa {

template <int D>
struct BkvCfg {
  static constexpr int BM = 128;                                     // resident keys
  static constexpr int BN = (D == 64) ? 128 : (D == 96 ? 96 : 64);   // streamed queries per tile
  static constexpr int CB = (D % 64 == 0) ? 64 : 32;                 // d column block (elements)
  static constexpr int SWZ = CB * 2;                                 // bytes per block row
  static constexpr int NCB = D / CB;
  static constexpr uint32_t LAYOUT = (SWZ == 128) ? 2u : 4u;
  static constexpr uint32_t SBO = 8u * SWZ;
  static constexpr uint32_t MBLOCK = (uint32_t)BM * SWZ;             // one d block of K or V
  static constexpr uint32_t M_BYTES = (uint32_t)BM * D * 2;
  static constexpr uint32_t NBLOCK = (uint32_t)BN * SWZ;             // one d block of Q or dO
  static constexpr uint32_t N_BYTES = (uint32_t)BN * D * 2;
  // P^T and dS^T: [BM keys][BN queries] in column blocks of CQ queries
  static constexpr int CQ = (BN % 64 == 0) ? 64 : 32;
  static constexpr int SWQ = CQ * 2;
  static constexpr uint32_t LAYOUT_Q = (SWQ == 128) ? 2u : 4u;
  static constexpr uint32_t SBO_Q = 8u * SWQ;
  static constexpr uint32_t QBLOCK = (uint32_t)BM * SWQ;
  static constexpr uint32_t PS_BYTES = (uint32_t)BM * BN * 2;
  static constexpr int NS = 3;
  static constexpr uint32_t STAGE_BYTES = 2 * N_BYTES;               // [Q | dO]
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = M_BYTES;                         // right after K (see dQ^T)
  static constexpr uint32_t OFF_ST = 2 * M_BYTES;
  static constexpr uint32_t OFF_P = OFF_ST + NS * STAGE_BYTES;
  static constexpr uint32_t OFF_DS = OFF_P + PS_BYTES;
  static constexpr uint32_t OFF_ROWV = OFF_DS + PS_BYTES;            // [NS][2][BN] fp32: lse log2 e, D
  static constexpr uint32_t OFF_BAR = OFF_ROWV + NS * 2 * BN * 4;
  // a ring slot holds a tile's [Q | dO] bf16, then its dQ^T as [BN][D] fp32
  static_assert(STAGE_BYTES == (uint32_t)BN * D * 4, "dQ staging fills one ring slot");
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
  // TMEM columns
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = BN;
  static constexpr int DV_COL = 2 * BN;
  static constexpr int DK_COL = 2 * BN + D;
  static constexpr int DQ_COL = 2 * BN + 2 * D;
  static constexpr int TMEM_COLS = 512;
  static_assert(DQ_COL + BN <= TMEM_COLS, "TMEM plan exceeds 512 columns");
  static_assert(MBLOCK % 1024 == 0 && NBLOCK % 1024 == 0 && QBLOCK % 1024 == 0 && M_BYTES % 1024 == 0 &&
                    N_BYTES % 1024 == 0 && PS_BYTES % 1024 == 0,
                "1 KB aligned tiles");
  // dQ^T reads 128 / CB d blocks from OFF_K: K's own, then the start of V
  static_assert(OFF_V == OFF_K + NCB * MBLOCK && (128 / CB) * MBLOCK <= 2 * M_BYTES, "K^T rows past d read V");
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);     // K-major A and B
  static constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);      // K-major A, MN-major B
  static constexpr uint32_t IDESC_Q = idesc_bf16(128, BN, 1, 1);     // MN-major A and B
  static constexpr int NSW = 16;                                     // P / dS warps (2..17)
  static constexpr int HC = BN / 4;                                  // columns per P / dS warp
  static constexpr int DQ_QUARTERS = (D + 31) / 32;                  // lane quarters with d rows of dQ^T
  static constexpr int NDRAIN = 4 * DQ_QUARTERS;                     // warps that stage dQ^T
  static constexpr int NUM_THREADS = 32 * (2 + NSW);
  static_assert(HC % 8 == 0 && HC >= 16 && HC <= 32, "whole 16-byte chunks per P / dS warp");
  static_assert(SMEM_BYTES <= 227u * 1024, "shared memory");
  // the epilogue's 32 x 33 fp32 staging slot per P / dS warp overlays K, V
  // and then P^T, dS^T (not the ring: the last tiles' reduce-adds may still
  // be reading their dQ^T rows there)
  static constexpr uint32_t EPI_SLOT = 32 * 33 * 4;
  static constexpr int EPI_KV_SLOTS = (int)(2 * M_BYTES / EPI_SLOT);
  static_assert((uint32_t)(NSW - EPI_KV_SLOTS) * EPI_SLOT <= 2 * PS_BYTES, "epilogue staging overlays K, V, P, dS");
};

enum : int {
  BK_RFULL = 0,      // K, V landed
  BK_FULL = 1,       // [3] ring slot landed
  BK_STG_FULL = 4,   // [3] count NDRAIN warps: the slot's dQ^T rows staged (its products are done)
  BK_SFULL = 7,      // S^T, dP^T of the current tile computed
  BK_SREAD = 8,      // count 16 warps: S^T, dP^T read into registers
  BK_PFULL = 9,      // count 16 warps: P^T, dS^T in shared memory (and the previous dQ^T read)
  BK_PEMPTY = 10,    // a tile's dV, dK, dQ^T products done (P^T, dS^T free; dQ^T ready)
  BK_DRAIN = 11,
  BK_TMEM_SLOT = 12,
  BK_ABORT_SLOT = 13,
};

__device__ __forceinline__ void bkv_tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}
// TMA reduce-add shared -> global (elements past the tensor map's bounds are
// dropped), tracked by this thread's bulk group.
__device__ __forceinline__ void bkv_tma_reduce_add_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2,
                                                      int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
      : "memory");
}
// N consecutive 32-bit TMEM columns of this warp's 32 lanes (N = 16, 24, 32)
template <int N>
__device__ __forceinline__ void bkv_tmem_ld(uint32_t taddr, uint32_t* r) {
  tmem_ld16(taddr, r);
  if constexpr (N == 32) tmem_ld16(taddr + 16, r + 16);
  if constexpr (N == 24) bkv_tmem_ld8(taddr + 16, r + 16);
}

// One CTA: keys r0 = 128 tile .. r0 + 127 of KV head g of sequence b.
template <int D>
__global__ void __launch_bounds__(BkvCfg<D>::NUM_THREADS, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BkvCfg<D>;
  constexpr int BN = C::BN;
  constexpr int HC = C::HC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * BK_TMEM_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * BK_ABORT_SLOT);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Blocks in order of key tile (tile 0, the one the most queries see, first)
  const int per_level = p.n_kv * p.B;
  const int tile = (int)blockIdx.x / per_level;
  const int g = ((int)blockIdx.x % per_level) % p.n_kv;
  const int b = ((int)blockIdx.x % per_level) / p.n_kv;
  const int r0 = tile * C::BM;
  // Query tiles [t_lo, t_hi) of BN rows that see keys r0..r0+127 (key j is
  // seen by queries j <= i < j + window), for each head of the group
  const int t_lo = r0 / BN;
  int i_end = p.T;
  if (p.window > 0 && r0 + C::BM - 1 + p.window < i_end) i_end = r0 + C::BM - 1 + p.window;
  const int t_hi = (i_end + BN - 1) / BN;
  const int per = t_hi > t_lo ? t_hi - t_lo : 0;
  const int n_tiles = per * p.q_mult;
  auto stream_of = [&](int u, int& hh, int& q0) {
    const int x = u / per;
    hh = g * p.q_mult + x;
    q0 = (t_lo + u - x * per) * BN;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(BK_RFULL), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BK_FULL + s), 1);
      mbar_init(bar(BK_STG_FULL + s), C::NDRAIN);
    }
    mbar_init(bar(BK_SFULL), 1);
    mbar_init(bar(BK_SREAD), C::NSW);
    mbar_init(bar(BK_PFULL), C::NSW);
    mbar_init(bar(BK_PEMPTY), 1);
    mbar_init(bar(BK_DRAIN), 1);
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
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(bar(BK_RFULL), 2 * C::M_BYTES);
#pragma unroll
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_4d(sbase + C::OFF_K + cb * C::MBLOCK, &tmK, bar(BK_RFULL), cb * C::CB, r0, g, b);
        tma_load_4d(sbase + C::OFF_V + cb * C::MBLOCK, &tmV, bar(BK_RFULL), cb * C::CB, r0, g, b);
      }
      // tile v's dQ^T rows, staged in its slot once its products were done,
      // added to dq
      auto reduce_tile = [&](int v) -> bool {
        const int sv = v % C::NS;
        if (!mbar_wait(bar(BK_STG_FULL + sv), (uint32_t)((v / C::NS) & 1))) return false;
        int hh, q0;
        stream_of(v, hh, q0);
        bkv_tma_reduce_add_4d(&tmDQ, sbase + C::OFF_ST + sv * C::STAGE_BYTES, 0, hh, q0, b);
        bulk_commit();
        return true;
      };
      int issued = 0;
      bool ok = true;
      for (int u = 0; u < n_tiles; ++u) {
        const int s = u % C::NS;
        if (u >= C::NS) {
          // the slot's previous tile: reduce its dQ^T rows, wait until they are read
          if (!reduce_tile(u - C::NS)) {
            ok = false;
            break;
          }
          bulk_wait_read_all();
        }
        if (*abort_flag) {
          ok = false;
          break;
        }
        int hh, q0;
        stream_of(u, hh, q0);
        mbar_arrive_expect_tx(bar(BK_FULL + s), C::STAGE_BYTES + 2 * BN * 4);
        // lse log2 e and D of the tile's BN query rows (padded workspace
        // rows: whole tiles, 16-byte aligned)
        const long long wb = ((long long)b * p.n_q + hh) * p.Tp + q0;
        const uint32_t rv = sbase + C::OFF_ROWV + s * 2 * BN * 4;
        bulk_load(rv, p.lse2 + wb, BN * 4, bar(BK_FULL + s));
        bulk_load(rv + BN * 4, p.dvec + wb, BN * 4, bar(BK_FULL + s));
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_BYTES;
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_4d(st + cb * C::NBLOCK, &tmQ, bar(BK_FULL + s), cb * C::CB, q0, hh, b);
          tma_load_4d(st + C::N_BYTES + cb * C::NBLOCK, &tmO, bar(BK_FULL + s), cb * C::CB, q0, hh, b);
        }
        issued = u + 1;
      }
      for (int v = (n_tiles > C::NS ? n_tiles - C::NS : 0); ok && v < n_tiles; ++v) ok = reduce_tile(v);
      // every reduce has read its rows and written dq before the CTA ends
      bulk_wait_all();
      if (!ok) {
        *abort_flag = 1;
        for (int u = (issued > C::NS ? issued - C::NS : 0); u < issued; ++u)
          mbar_wait_drain(bar(BK_FULL + u % C::NS), (uint32_t)((u / C::NS) & 1));
      }
      mbar_wait_drain(bar(BK_RFULL), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(BK_RFULL), 0);
      tc_fence_after();
      const uint64_t a_k = smem_desc(sbase + C::OFF_K, 16, C::SBO, C::LAYOUT);        // K, K-major
      const uint64_t a_v = smem_desc(sbase + C::OFF_V, 16, C::SBO, C::LAYOUT);        // V, K-major
      const uint64_t a_kt = smem_desc(sbase + C::OFF_K, C::MBLOCK, C::SBO, C::LAYOUT); // K^T, MN-major
      const uint64_t a_p = smem_desc(sbase + C::OFF_P, 16, C::SBO_Q, C::LAYOUT_Q);   // P^T, K-major
      const uint64_t a_ds = smem_desc(sbase + C::OFF_DS, 16, C::SBO_Q, C::LAYOUT_Q); // dS^T, K-major
      const uint64_t b_ds = smem_desc(sbase + C::OFF_DS, C::QBLOCK, C::SBO_Q, C::LAYOUT_Q);  // dS^T, MN-major
      // tile v's dV += P^T dO, dK += dS^T Q (K = BN queries) and dQ^T = K^T dS^T (K = 128 keys)
      auto products = [&](int v) {
        const int sv = v % C::NS;
        const uint32_t st = sbase + C::OFF_ST + sv * C::STAGE_BYTES;
        const uint64_t b_q = smem_desc(st, C::NBLOCK, C::SBO, C::LAYOUT);              // Q, MN-major
        const uint64_t b_o = smem_desc(st + C::N_BYTES, C::NBLOCK, C::SBO, C::LAYOUT); // dO, MN-major
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t aoff = ((uint32_t)(kk * 16 / C::CQ) * C::QBLOCK + (uint32_t)(kk * 16 % C::CQ) * 2) >> 4;
          const uint32_t boff = ((uint32_t)kk * 16 * C::SWZ) >> 4;
          const uint32_t acc = (v > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem + C::DV_COL, a_p + aoff, b_o + boff, C::IDESC_O, acc);
          mma_ss(tmem + C::DK_COL, a_ds + aoff, b_q + boff, C::IDESC_O, acc);
        }
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          mma_ss(tmem + C::DQ_COL, a_kt + (((uint32_t)kk * 16 * C::SWZ) >> 4),
                 b_ds + (((uint32_t)kk * 16 * C::SWQ) >> 4), C::IDESC_Q, kk > 0 ? 1u : 0u);
        mma_commit(bar(BK_PEMPTY));
      };
      for (int u = 0; u < n_tiles && ok; ++u) {
        const int s = u % C::NS;
        if (!mbar_wait(bar(BK_FULL + s), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
        // the warps have read the previous tile's S^T, dP^T
        if (u >= 1 && !mbar_wait(bar(BK_SREAD), (uint32_t)((u - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_BYTES;
        const uint64_t b_q = smem_desc(st, 16, C::SBO, C::LAYOUT);                // Q, K-major
        const uint64_t b_o = smem_desc(st + C::N_BYTES, 16, C::SBO, C::LAYOUT);   // dO, K-major
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t cb = kk * 16 / C::CB, cin = (kk * 16 % C::CB) * 2;
          mma_ss(tmem + C::S_COL, a_k + ((cb * C::MBLOCK + cin) >> 4), b_q + ((cb * C::NBLOCK + cin) >> 4),
                 C::IDESC_S, kk > 0 ? 1u : 0u);
          mma_ss(tmem + C::DP_COL, a_v + ((cb * C::MBLOCK + cin) >> 4), b_o + ((cb * C::NBLOCK + cin) >> 4),
                 C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BK_SFULL));
        if (u >= 1) {
          if (!mbar_wait(bar(BK_PFULL), (uint32_t)((u - 1) & 1))) { ok = false; break; }
          tc_fence_after();
          products(u - 1);
        }
        if (*abort_flag) { ok = false; break; }
      }
      if (ok && n_tiles > 0) {
        if (mbar_wait(bar(BK_PFULL), (uint32_t)((n_tiles - 1) & 1))) {
          tc_fence_after();
          products(n_tiles - 1);
        } else {
          ok = false;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(bar(BK_DRAIN));
        mbar_wait_drain(bar(BK_DRAIN), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ and the epilogue
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;                    // which HC columns of a tile
    const int rr = quarter * 32 + lane;                  // resident key row of this thread
    const int key = r0 + rr;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int c_base = part * HC;
    const float sl2 = p.scale_log2;
    // every wait below is taken warp-uniformly: the TMEM loads that follow
    // are warp-collective
    auto wait_all = [&](uint32_t bb, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bb, parity) ? 1 : 0) != 0;
    };
    // dQ^T of finished tile v -> [query][d] fp32 rows in its ring slot
    // (lane = d row: each store covers 32 consecutive words), reduced into dq
    // by the TMA thread
    auto drain_dq = [&](int v) {
      if (quarter >= C::DQ_QUARTERS) return;
      float* stg = reinterpret_cast<float*>(smem + C::OFF_ST + (v % C::NS) * C::STAGE_BYTES);
      const int dcol = quarter * 32 + lane;
#pragma unroll
      for (int c0 = 0; c0 < HC; c0 += 8) {   // eight columns per TMEM load (few live registers)
        uint32_t qv[8];
        bkv_tmem_ld8(tmem + lane_base + C::DQ_COL + c_base + c0, qv);
        tmem_wait_ld();
        if (dcol < D) {
#pragma unroll
          for (int c = 0; c < 8; ++c) stg[(c_base + c0 + c) * D + dcol] = __uint_as_float(qv[c]) * p.scale;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BK_STG_FULL + v % C::NS));
    };
    bool ok = true;
    for (int u = 0; u < n_tiles && ok; ++u) {
      if (!wait_all(bar(BK_SFULL), (uint32_t)(u & 1))) { ok = false; break; }
      tc_fence_after();
      int hh, q0;
      stream_of(u, hh, q0);
      uint32_t sv[HC], dv[HC];
      bkv_tmem_ld<HC>(tmem + lane_base + C::S_COL + c_base, sv);
      bkv_tmem_ld<HC>(tmem + lane_base + C::DP_COL + c_base, dv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BK_SREAD));
      // the stage's lse / D values: acquired on the stage's own barrier (its
      // phase cannot move on before this tile's products, which wait for
      // these warps)
      if (!wait_all(bar(BK_FULL + u % C::NS), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
      const float* rv = reinterpret_cast<const float*>(smem + C::OFF_ROWV) + (u % C::NS) * 2 * BN;
      // every (key, query) pair of the tile admitted? (pairs past T are
      // harmless either way: their operand rows are zero or their output
      // rows are not stored)
      const bool all_in = r0 + C::BM - 1 <= q0 && (p.window <= 0 || r0 > q0 + BN - 1 - p.window);
      uint32_t pk[HC / 2], dk[HC / 2];
      float4 lv4 = make_float4(0.f, 0.f, 0.f, 0.f), dv4 = lv4;
#pragma unroll
      for (int c = 0; c < HC; c += 2) {
        if ((c & 3) == 0) {   // the tile's per-column lse / D, four at a time
          lv4 = *reinterpret_cast<const float4*>(rv + c_base + c);
          dv4 = *reinterpret_cast<const float4*>(rv + BN + c_base + c);
        }
        const float l0 = (c & 3) ? lv4.z : lv4.x, l1 = (c & 3) ? lv4.w : lv4.y;
        const float d0 = (c & 3) ? dv4.z : dv4.x, d1 = (c & 3) ? dv4.w : dv4.y;
        float p0, p1;
        fma2(p0, p1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl2, sl2, -l0, -l1);
        // every other pair on the FMA pipe (the degree-3 exp2 of the
        // forward, relative error < 1.5e-4), the rest on the MUFU unit
        // (measured: all on MUFU 0.974 ms, one in four on the FMA pipe 0.965,
        // one in two 0.953 on the Lite full-causal layer)
        if (((c / 2) & 1) == 0) {
          exp2_fma2(p0, p1);
        } else {
          p0 = ex2(p0);
          p1 = ex2(p1);
        }
        if (!all_in) {
          const int qi = q0 + c_base + c;
          if (!bwd_admitted(qi, key, p.T, p.window)) p0 = 0.f;
          if (!bwd_admitted(qi + 1, key, p.T, p.window)) p1 = 0.f;
        }
        float t0 = __uint_as_float(dv[c]), t1 = __uint_as_float(dv[c + 1]);
        add2(t0, t1, -d0, -d1);
        mul2(t0, t1, p0, p1);
        pk[c / 2] = pack_bf16(p0, p1);
        dk[c / 2] = pack_bf16(t0, t1);
      }
      if (u >= 1) {
        // the previous tile's products are done: its P^T, dS^T buffers are
        // free and its dQ^T is final
        if (!wait_all(bar(BK_PEMPTY), (uint32_t)((u - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        drain_dq(u - 1);
      }
      // P^T, dS^T rows (this thread's key row, columns c_base..) in 16-byte
      // chunks of the swizzled layout the products read
#pragma unroll
      for (int j = 0; j < HC / 8; ++j) {
        const uint32_t off = swz_off<C::CQ>(rr, c_base + 8 * j, C::QBLOCK);
        *reinterpret_cast<uint4*>(smem + C::OFF_P + off) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        *reinterpret_cast<uint4*>(smem + C::OFF_DS + off) =
            make_uint4(dk[4 * j], dk[4 * j + 1], dk[4 * j + 2], dk[4 * j + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BK_PFULL));
      if (*abort_flag) { ok = false; break; }
    }
    // the last tile's products (the accumulators are then final too)
    const bool have = n_tiles > 0;
    if (ok && have) {
      if (wait_all(bar(BK_PEMPTY), (uint32_t)((n_tiles - 1) & 1))) {
        tc_fence_after();
        drain_dq(n_tiles - 1);
      } else {
        ok = false;
      }
    }
    // epilogue: dV (the first two warps of each quarter) and dK (the other
    // two) -> fp32 rows, 32-column chunks in turn. Every lane takes part in
    // the TMEM loads; rows past T store nothing.
    if (ok) {
      const bool is_dv = part < 2;
      float* out = (is_dv ? p.dv : p.dk) + ((long long)b * p.T * p.n_kv + g) * D;
      const long long rstride = (long long)p.n_kv * D;
      const float mul = is_dv ? 1.0f : p.scale;
      const int acc = is_dv ? C::DV_COL : C::DK_COL;
      // Each 32 x 32 chunk (this warp's 32 rows) is transposed through shared
      // memory so that every store instruction writes one row's 128 bytes.
      // The staging slots overlay K, V and P^T, dS^T, which every product
      // has finished reading once the last PEMPTY phase has completed (with
      // no tile there is no such wait: zeros are stored directly).
      const int es = warp - 2;
      float* stg = reinterpret_cast<float*>(
          smem + (es < C::EPI_KV_SLOTS ? C::OFF_K + es * C::EPI_SLOT : C::OFF_P + (es - C::EPI_KV_SLOTS) * C::EPI_SLOT));
      const int krow0 = r0 + quarter * 32;   // first key row of this warp's quarter
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        if ((c0 / 32) % 2 != part % 2) continue;
        if (have) {
          uint32_t a32[32];
          tmem_ld32(tmem + lane_base + acc + c0, a32);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) stg[lane * 33 + c] = __uint_as_float(a32[c]) * mul;
          __syncwarp();
#pragma unroll 4
          for (int r = 0; r < 32; ++r)
            if (krow0 + r < p.T) out[(long long)(krow0 + r) * rstride + c0 + lane] = stg[r * 33 + lane];
          __syncwarp();
        } else {
          for (int r = 0; r < 32; ++r)
            if (krow0 + r < p.T) out[(long long)(krow0 + r) * rstride + c0 + lane] = 0.f;
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

}  // namespace sa
