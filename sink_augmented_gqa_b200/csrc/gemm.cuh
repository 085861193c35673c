// The dense projections around the attention, as one persistent tcgen05 GEMM
// with fused prologue / epilogue work (GQA Attention study note, "How it
// works": pre-norm RMSNorm, the fused linear qkv of width d_h (n_q + 2 n_kv),
// and after attention the linear out back to the residual width with the
// residual add; both linears bf16 with bias):
//
//   y[m][n] = s_m * sum_k a[m][k] w[n][k] + bias[n] (+ residual[m][n])
//
// with s_m = 1 / sqrt(mean_k a[m][k]^2 + eps) for the qkv projection (the
// RMSNorm gain gamma is folded into w once, w[n][k] * gamma[k], so the
// normalised activations are never materialised) and s_m = 1 for the out
// projection, whose epilogue adds the residual (x <- x + out(o), in place).
//
// One CTA per SM walks 256 x 256 output tiles (tile t, t + grid, ...):
//
//   warp 0      TMA producer: per 64-wide K step, the A tile (256 x 64) and
//               the W tile (256 x 64), 128-byte swizzled, into a 3-deep ring.
//   warp 1      one thread issues tcgen05.mma (kind::f16, M 128, N 256, K 16
//               per instruction, fp32 accumulation in TMEM): two products per
//               K step, rows 0-127 and 128-255 of A against the same W tile
//               (131 flops per operand byte instead of 87 with one), into the
//               two 256-column halves of TMEM.
//   warps 2, 3  (RMSNorm only) sum the squares of each A row from the same
//               shared-memory tiles the tensor core reads, and publish s_m.
//   warps 4-11  epilogue, one output row per thread (warp 4 + 4 h + q reads
//               TMEM lanes 32 q.. of half h): per 32-column chunk,
//               tcgen05.ld, scale, bias, residual, bf16, staged in shared
//               memory (64-byte swizzle) and written by a TMA tile store
//               (which clips the ragged edges of M and N). The accumulator is
//               single-buffered: the next tile's products wait for this
//               drain (a few per cent of a tile's main loop).
#pragma once

#include "ptx.cuh"

namespace sa {

struct GemmParams {
  int M, N, K;
  const __nv_bfloat16* bias;      // [N] or null
  const __nv_bfloat16* residual;  // [M] rows of ldr elements, or null; may alias the output
  long long ldr;
  int rms;                        // 1: scale row m by 1 / sqrt(mean_k a^2 + eps)
  float eps;
  int tiles_m, tiles_n;
};

// BN_: output columns per tile (256); the two accumulator halves sit at TMEM
// columns 0 and 256.
template <int BN_>
struct GemmCfg {
  static constexpr int BM = 256, BN = BN_, BK = 64;
  static constexpr int NS = 3;                               // ring depth
  static constexpr uint32_t A_BYTES = BM * BK * 2;           // 32 KB
  static constexpr uint32_t A_HALF = 128 * BK * 2;           // rows 128.. of the A tile
  static constexpr uint32_t B_BYTES = BN * BK * 2;           // 32 KB
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = NS * A_BYTES;
  static constexpr int EPI_WARPS = 8;
  static constexpr uint32_t OFF_ST = OFF_B + NS * B_BYTES;   // [8 warps][2] 32 rows x 64 B
  static constexpr uint32_t ST_BYTES = 32 * 64;
  static constexpr uint32_t OFF_RMS = OFF_ST + EPI_WARPS * 2 * ST_BYTES;   // [256] fp32 row scales
  static constexpr uint32_t OFF_BAR = OFF_RMS + BM * 4;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per block");
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC = idesc_bf16(128, BN, 0, 0);
  static constexpr uint32_t SBO = 1024;                      // 8 rows x 128 B
  static constexpr uint32_t HALF_COL = 256;                  // TMEM column of accumulator half 1
  static constexpr int NUM_THREADS = 32 * (4 + EPI_WARPS);
  static_assert(BN % 32 == 0 && BN <= 256, "whole 32-column epilogue chunks");
  static_assert(OFF_B % 1024 == 0 && OFF_ST % 1024 == 0 && A_HALF % 1024 == 0 && B_BYTES % 1024 == 0,
                "swizzled buffers need 1 KB alignment");
};

enum : int {
  GB_FULL = 0,        // [NS] producer -> MMA, RMS warps: A and W tiles landed
  GB_EMPTY = 4,       // [NS] MMA (commit) + the 64 RMS lanes -> producer
  GB_ACC_FULL = 8,    // MMA -> epilogue: the tile's accumulator is complete
  GB_ACC_EMPTY = 10,  // count 8: epilogue warps -> MMA: accumulator read
  GB_RMS_FULL = 12,   // count 64: RMS lanes -> epilogue: row scales of the tile
  GB_RMS_EMPTY = 14,  // count 8: epilogue warps -> RMS warps
  GB_DRAIN = 16,      // MMA issuer, on abort
  GB_TMEM_SLOT = 17,
  GB_ABORT_SLOT = 18,
};

__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

template <int BN_>
__global__ void __launch_bounds__(384, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  using C = GemmCfg<BN_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * GB_TMEM_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * GB_ABORT_SLOT);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = p.tiles_m * p.tiles_n;
  const int n_kb = (p.K + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(GB_FULL + s), 1);
      mbar_init(bar(GB_EMPTY + s), p.rms ? 65 : 1);   // MMA commit (+ one arrival per RMS lane)
    }
    mbar_init(bar(GB_ACC_FULL), 1);
    mbar_init(bar(GB_ACC_EMPTY), C::EPI_WARPS);
    mbar_init(bar(GB_RMS_FULL), 64);
    mbar_init(bar(GB_RMS_EMPTY), C::EPI_WARPS);
    mbar_init(bar(GB_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // output tiles walk N fastest: the ~grid tiles in flight at a time cover all
  // of W and a band of grid / tiles_n row tiles of A, which together stay in L2
  // (every A row is read from DRAM once; W once per pass over it)
  auto tile_origin = [&](int t, int& m0, int& n0) {
    n0 = (t % p.tiles_n) * C::BN;
    m0 = (t / p.tiles_n) * C::BM;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int m0, n0;
        tile_origin(t, m0, n0);
        for (int kb = 0; kb < n_kb; ++kb) {
          const int s = it % C::NS;
          const uint32_t ph = (uint32_t)((it / C::NS) & 1);
          if (it >= C::NS && !mbar_wait(bar(GB_EMPTY + s), ph ^ 1)) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          mbar_arrive_expect_tx(bar(GB_FULL + s), C::A_BYTES + C::B_BYTES);
          tma_load_4d(sbase + C::OFF_A + s * C::A_BYTES, &tmA, bar(GB_FULL + s), kb * C::BK, m0, 0, 0);
          tma_load_4d(sbase + C::OFF_B + s * C::B_BYTES, &tmB, bar(GB_FULL + s), kb * C::BK, n0, 0, 0);
          ++it;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // let every copy still in flight land before the CTA can exit
        for (int u = (it > C::NS ? it - C::NS : 0); u < it; ++u)
          mbar_wait_drain(bar(GB_FULL + u % C::NS), (uint32_t)((u / C::NS) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint64_t ad0 = smem_desc(sbase + C::OFF_A, 16, C::SBO, 2u);
      const uint64_t bd0 = smem_desc(sbase + C::OFF_B, 16, C::SBO, 2u);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tl) {
        // the accumulator (both halves) has been drained by the previous tile's epilogue
        if (tl >= 1 && !mbar_wait(bar(GB_ACC_EMPTY), (uint32_t)((tl - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < n_kb; ++kb, ++it) {
          const int s = it % C::NS;
          if (!mbar_wait(bar(GB_FULL + s), (uint32_t)((it / C::NS) & 1))) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = ad0 + ((uint32_t)(s * C::A_BYTES) >> 4);
          const uint64_t bd = bd0 + ((uint32_t)(s * C::B_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {   // 32 bytes further along the swizzled rows
            mma_ss(tmem, ad + 2 * kk, bd + 2 * kk, C::IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_ss(tmem + C::HALF_COL, ad + (C::A_HALF >> 4) + 2 * kk, bd + 2 * kk, C::IDESC,
                   (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(GB_EMPTY + s));
        }
        if (!ok) break;
        mma_commit(bar(GB_ACC_FULL));
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(bar(GB_DRAIN));
        mbar_wait_drain(bar(GB_DRAIN), 0);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ RMSNorm row scales
    // Every lane waits and arrives on its own (the barriers count 64 RMS
    // arrivals): there is no warp-collective step, so a wait that runs out in
    // one lane cannot leave the others waiting for it.
    if (p.rms) {
      const int rb0 = 32 * (warp - 2) + lane;   // rows rb0 + 64 i of the A tile, i < 4
      const float inv_k = 1.0f / (float)p.K;
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tl) {
        float ss[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = 0; kb < n_kb; ++kb, ++it) {
          const int s = it % C::NS;
          if (!mbar_wait(bar(GB_FULL + s), (uint32_t)((it / C::NS) & 1))) { ok = false; break; }
          const uint8_t* a = smem + C::OFF_A + s * C::A_BYTES;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = rb0 + 64 * i;
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // 16-byte chunk j of a row sits at chunk j ^ (row % 8)
              const uint4 u = *reinterpret_cast<const uint4*>(a + r * 128 + ((j ^ (r & 7)) << 4));
              const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a0 = bf16_lo(w[e]), a1 = bf16_hi(w[e]);
                ss[i] = fmaf(a0, a0, fmaf(a1, a1, ss[i]));
              }
            }
          }
          mbar_arrive(bar(GB_EMPTY + s));
        }
        if (!ok) break;
        if (tl >= 1 && !mbar_wait(bar(GB_RMS_EMPTY), (uint32_t)((tl - 1) & 1))) { ok = false; break; }
        float* rb = reinterpret_cast<float*>(smem + C::OFF_RMS);
#pragma unroll
        for (int i = 0; i < 4; ++i) rb[rb0 + 64 * i] = 1.0f / sqrtf(ss[i] * inv_k + p.eps);
        mbar_arrive(bar(GB_RMS_FULL));
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int hh = (warp - 4) >> 2;          // accumulator half: rows 128 hh ..
    const int r = 128 * hh + 32 * q + lane;  // row within the tile
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // warp-uniform waits: the TMEM loads and __syncwarp that follow are
    // warp-collective
    auto wait_all = [&](uint32_t bb, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bb, parity) ? 1 : 0) != 0;
    };
    int tl = 0, cnt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tl) {
      int m0, n0;
      tile_origin(t, m0, n0);
      if (!wait_all(bar(GB_ACC_FULL), (uint32_t)(tl & 1))) { ok = false; break; }
      tc_fence_after();
      float sc = 1.f;
      if (p.rms) {
        if (!wait_all(bar(GB_RMS_FULL), (uint32_t)(tl & 1))) { ok = false; break; }
        sc = reinterpret_cast<const float*>(smem + C::OFF_RMS)[r];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(GB_RMS_EMPTY));
      }
      const int m = m0 + r;
      const bool row_ok = m < p.M;
      const int nch = min(C::BN / 32, (p.N - n0 + 31) / 32);
      for (int c = 0; c < nch; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(hh * C::HALF_COL + 32 * c), v);
        tmem_wait_ld();
        const int nb = n0 + 32 * c;
        const bool full = nb + 32 <= p.N;
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(v[j]) * sc;
        if (p.bias) {
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const uint4 bv = __ldg(reinterpret_cast<const uint4*>(p.bias + nb + j));
              y[j + 0] += bf16_lo(bv.x); y[j + 1] += bf16_hi(bv.x);
              y[j + 2] += bf16_lo(bv.y); y[j + 3] += bf16_hi(bv.y);
              y[j + 4] += bf16_lo(bv.z); y[j + 5] += bf16_hi(bv.z);
              y[j + 6] += bf16_lo(bv.w); y[j + 7] += bf16_hi(bv.w);
            }
          } else {
            for (int j = 0; j < 32; ++j)
              if (nb + j < p.N) y[j] += __bfloat162float(p.bias[nb + j]);
          }
        }
        if (p.residual && row_ok) {
          const __nv_bfloat16* rr = p.residual + (long long)m * p.ldr + nb;
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const uint4 rv = *reinterpret_cast<const uint4*>(rr + j);
              y[j + 0] += bf16_lo(rv.x); y[j + 1] += bf16_hi(rv.x);
              y[j + 2] += bf16_lo(rv.y); y[j + 3] += bf16_hi(rv.y);
              y[j + 4] += bf16_lo(rv.z); y[j + 5] += bf16_hi(rv.z);
              y[j + 6] += bf16_lo(rv.w); y[j + 7] += bf16_hi(rv.w);
            }
          } else {
            for (int j = 0; j < 32; ++j)
              if (nb + j < p.N) y[j] += __bfloat162float(rr[j]);
          }
        }
        // stage the 32 x 32 chunk of this warp (64-byte rows, 64-byte swizzle:
        // 16-byte chunk j of row r at j ^ ((r / 2) % 4)) and store it by TMA
        const int sb = cnt & 1;
        uint8_t* st = smem + C::OFF_ST + (uint32_t)((warp - 4) * 2 + sb) * C::ST_BYTES;
        if (cnt >= 2) {
          if (lane == 0) bulk_wait_read_1();   // the store that last used this buffer has read it
          __syncwarp();
        }
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          uint4 w;
          w.x = pack_bf16(y[8 * j4 + 0], y[8 * j4 + 1]);
          w.y = pack_bf16(y[8 * j4 + 2], y[8 * j4 + 3]);
          w.z = pack_bf16(y[8 * j4 + 4], y[8 * j4 + 5]);
          w.w = pack_bf16(y[8 * j4 + 6], y[8 * j4 + 7]);
          *reinterpret_cast<uint4*>(st + lane * 64 + ((j4 ^ ((lane >> 1) & 3)) << 4)) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int row0 = m0 + 128 * hh + 32 * q;
          if (row0 < p.M)   // rows past M are clipped; a wholly outside chunk is not stored
            tma_store_4d(&tmC, smem_u32(st), nb, row0, 0, 0);
          bulk_commit();
        }
        ++cnt;
      }
      // the accumulator is free for the next tile's products
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(GB_ACC_EMPTY));
      if (*abort_flag) { ok = false; break; }
    }
    if (lane == 0) bulk_wait_all();   // output stores complete before the CTA exits
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

// w_folded[n][k] = bf16(w[n][k] * gamma[k]), the product formed exactly in
// fp64 and rounded once (RMSNorm's gain folded into the qkv weight).
__global__ void fold_gamma_kernel(const __nv_bfloat16* __restrict__ w, long long ldw,
                                  const float* __restrict__ gamma, __nv_bfloat16* __restrict__ out,
                                  long long ldo, int N, int K) {
  const long long n_el = (long long)N * K;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n_el;
       idx += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(idx / K), k = (int)(idx % K);
    const double prod = (double)__bfloat162float(w[n * ldw + k]) * (double)gamma[k];
    out[n * ldo + k] = __ushort_as_bfloat16((unsigned short)bf16_bits_from_f64(prod));
  }
}

}  // namespace sa
