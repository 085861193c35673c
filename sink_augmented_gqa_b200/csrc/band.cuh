// Band-layer prefill (keys p-W+1 .. p, W small) on tcgen05 tensor cores,
// with the query heads of a KV group packed into the MMA rows.
//
// GQA Attention study note, "How it works": a band row attends to at most W
// keys, and every query head of a KV group reads the same keys. A unit of
// work is one (sequence b, KV head g) and R = 128 / q_mult consecutive query
// positions i0 .. i0+R-1: its 128 MMA rows are those positions times the
// group's q_mult heads (row m = r q_mult + head), so the key window that
// serves all of them is only R + W - 1 keys wide (plus up to 15 to start on
// a multiple of 16): 160 columns for q_mult = 8, W = 128, of which 128 per
// row are admitted, against 256 with 128-row single-head query tiles. Every
// row sees all of its keys in that one tile, so the softmax is a single pass
// (max, then exp2 and sum) with no running rescale, seeded with the sink.
//
// Queries come straight from q and are rotated in shared memory by the
// softmax warps of the unit (correctly rounded bf16, as the staged copy would
// be); K and V are read from the cache, which the staging launch before this
// one has appended to (K rotated).
//
//   warp 0      TMA producer: per unit the Q box (d x q_mult heads x R rows,
//               rows past T read as zeros) and the K and V windows (one box
//               each, negative positions read as zeros; a window that wraps
//               around a ring cache as 16-row boxes starting on multiples of
//               16 positions) into an NS-deep ring of stages.
//   warps 1, 2  one thread each issues the MMAs of pipeline X (the CTA's
//               units alternate between two pipelines): S_X = Q K^T (smem x
//               smem), then O_X = P_X V with P_X bf16 in TMEM over S_X.
//               Warp 1 owns the TMEM allocation.
//   warp 3      one thread stores each unit's output box with a TMA tile
//               store from the stage's Q area and releases the stage.
//   warps 4-11  pipeline 0, warps 12-19 pipeline 1: two threads per MMA row
//               (TMEM lane = row), each with half of the row's key columns:
//               RoPE of its half of the query row, mask, max (traded with
//               the other half), exp2, P -> TMEM, then O / l -> bf16 into the
//               stage.
//
// TMEM (512 columns): pipeline X has S_X at 256 X (N <= 160 columns; P of
// each 16-column chunk packed over the chunk's first 8 columns), O_X at
// 256 X + 160 (d = 64 columns) and 8 columns after it for the halves' trade.
#pragma once

#include "prefill.cuh"
#include "rope.cuh"

namespace sa {

struct BandParams {
  float* lse;
  const float* sinks;
  const float* cos_t;
  const float* sin_t;
  int B, T, n_q, n_kv, q_mult;
  long long off;
  int window;
  float scale_log2;
  int rope;
  int ring_cap;   // 0: cache row = position; > 0: ring cache, row = position mod ring_cap
  int R;          // query positions per unit (128 / q_mult)
  int N;          // key columns per unit: a multiple of 32, at most 160
  int n_blk;      // units per (b, g): ceil(T / R)
  int n_units;    // B * n_kv * n_blk
};

template <int D>
struct BandCfg {
  static_assert(D == 64, "the band kernel is built for d = 64 (one 128-byte swizzle row per row)");
  static constexpr int NMAX = 160;
  static constexpr uint32_t ROWB = D * 2;                   // 128 bytes
  static constexpr uint32_t Q_BYTES = 128u * ROWB;          // 16 KB
  static constexpr uint32_t KV_BYTES = (uint32_t)NMAX * ROWB;  // 20 KB
  static constexpr uint32_t OFF_K = Q_BYTES;
  static constexpr uint32_t OFF_V = Q_BYTES + KV_BYTES;
  static constexpr uint32_t STAGE_BYTES = Q_BYTES + 2 * KV_BYTES;
  // four stages: each pipeline has a unit in work and the next one loading
  // while the store of the unit before still holds its stage
  static constexpr int NS = 4;
  static constexpr uint32_t OFF_BAR = NS * STAGE_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
  static constexpr int NUM_THREADS = 544;
  static constexpr uint32_t SBO = 8u * ROWB;                // 8-row core-matrix group stride
  static constexpr uint32_t LAYOUT = 2u;                    // 128-byte swizzle
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL1 = 256;
  static constexpr int O_OFF = NMAX;                        // O_X = S_X + NMAX
  static constexpr int XCH_OFF = NMAX + D;                  // 2 x 4 columns for the halves' max / sum
  static_assert(XCH_OFF + 8 <= S_COL1, "a pipeline's TMEM columns fit in 256");
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 0, 1);
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "1 KB aligned tiles");
  static_assert(NS <= 4 && SMEM_BYTES <= 232448, "stages and barriers fit the shared memory of one CTA");
};

// Barrier slots (8 bytes each) at OFF_BAR.
enum : int {
  BD_FULL = 0,     // [NS <= 4] producer (TMA) -> pipelines: the unit's Q, K, V landed
  BD_EMPTY = 4,    // [NS] store thread -> producer: the stage's output box has been read
  BD_QROT = 8,     // [2] pipeline X's 4 warps -> MMA X: Q rotated in smem
  BD_SFULL = 10,   // [2] MMA X -> pipeline X: S_X computed
  BD_PFULL = 12,   // [2] pipeline X's 4 warps -> MMA X: P_X stored
  BD_ODONE = 14,   // [2] MMA X -> pipeline X: O_X = P_X V completed
  BD_EPI = 16,     // [2] pipeline X's 4 warps -> store thread: O staged in smem
  BD_DRAIN = 18,   // [2] per MMA issuer, on abort
  BD_TMEM_SLOT = 20,
  BD_ABORT_SLOT = 21,
};

// Unit u -> (b, g, first query row i0); units of one (b, g) are adjacent so
// that CTAs running side by side share most of their K/V windows in L2.
__device__ __forceinline__ void band_unit(const BandParams& p, int u, int& b, int& g, int& i0) {
  const int blk = u % p.n_blk, rest = u / p.n_blk;
  g = rest % p.n_kv;
  b = rest / p.n_kv;
  i0 = blk * p.R;
}
// First key position of the unit's window: a multiple of 16 at or below
// off + i0 - W + 1 (may be negative; those keys are masked and read as zeros).
__device__ __forceinline__ int band_window_start(const BandParams& p, int i0) {
  return floordiv((int)p.off + i0 - p.window + 1, 16) * 16;
}

// Pipeline X's eight warps (warps 1-8 or 9-16): two threads per MMA row m
// (= TMEM lane; both warps of a lane quarter hold the same rows), holding
// query position i0 + m / q_mult of head g q_mult + m % q_mult; half hf of
// the pair takes key columns [hf N/2, (hf+1) N/2), RoPE dims 16 hf .. 16 hf
// + 15 (and their partners), and output dims 32 hf .. 32 hf + 31. The two
// halves trade their row maxima and sums through spare TMEM columns.
// The queries of a pipeline's next unit are rotated while the tensor core
// computes the current unit's O = P V.
template <int D>
__device__ __forceinline__ void band_softmax(const BandParams& p, uint8_t* smem, uint32_t bar0, uint32_t tmem,
                                             volatile int* abort_flag, int warp, int lane) {
  using C = BandCfg<D>;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  const int X = (warp - 1) >> 3;
  const int hf = ((warp - 1) >> 2) & 1;
  const int quarter = warp & 3;                 // TMEM lane quarter a warp may access: warp % 4
  const int m = quarter * 32 + lane;
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const uint32_t s_tm = tmem + lane_base + (X ? C::S_COL1 : 0);
  const uint32_t o_tm = s_tm + C::O_OFF;
  // [max h0, max h1, sum h0, sum h1] per unit parity: a half writes the next
  // unit's values while the other may still read this unit's
  const uint32_t x_tm0 = s_tm + C::XCH_OFF;
  const int QM = p.q_mult;
  const int r = m / QM, hq = m - r * QM;
  const int G = gridDim.x;
  const float LOG2E = 1.4426950408889634f, LN2 = 0.6931471805599453f;
  const float scale = p.scale_log2;
  const int nh = p.N / 32;                      // 16-column chunks per half
  const int j0 = hf * nh;                       // first chunk of this half
  const uint32_t swz = (uint32_t)(m & 7);       // 128-byte swizzle: chunk c of row m sits at c ^ (m % 8)
  const int pipe_bar = 1 + X;                   // named barrier of the pipeline's 256 threads

  // Waits that run out (or any after the CTA aborted) are skipped, not left:
  // the pipeline's threads leave the loop together, at the trade of maxima,
  // so none is left waiting at that barrier.
  bool fail = false;
  // RoPE of this half of the row's query of unit k at its position (rows past
  // T are zeros and are not rotated: their positions may lie past the
  // tables), then this warp's arrival on Q_ROTATED.
  auto rotate_unit = [&](int k) {
    const int u = blockIdx.x + k * G;
    int b, g, i0;
    band_unit(p, u, b, g, i0);
    const int qp = (int)p.off + i0 + r;
    const bool rot = p.rope && i0 + r < p.T;
    const int s = k % C::NS;
    fail = fail || *abort_flag || !mbar_wait(bar(BD_FULL + s), (uint32_t)((k / C::NS) & 1));
    if (rot) {
      uint8_t* qrow = smem + (size_t)s * C::STAGE_BYTES + (size_t)m * C::ROWB;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {   // chunk c = 2 hf + cc (dims 8c ..) pairs with chunk c + D/16
        const uint32_t c = (uint32_t)(2 * hf + cc);
        uint4* pa = reinterpret_cast<uint4*>(qrow + ((c ^ swz) << 4));
        uint4* pb = reinterpret_cast<uint4*>(qrow + (((c + D / 16) ^ swz) << 4));
        uint4 a = *pa, bb = *pb;
        rotate8(a, bb, p.cos_t + (long long)qp * (D / 2) + 8 * c, p.sin_t + (long long)qp * (D / 2) + 8 * c);
        *pa = a;
        *pb = bb;
      }
      fence_proxy_async_smem();   // the tensor core reads the rotated rows through the async proxy
    }
    tc_fence_before();   // this warp's earlier TMEM reads and writes are done
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(BD_QROT + X));
  };

  int n = 0;
  if (blockIdx.x + X * G < p.n_units) rotate_unit(X);
  for (int k = X;; k += 2, ++n) {
    const int u = blockIdx.x + k * G;
    if (u >= p.n_units) break;
    const int s = k % C::NS;
    int b, g, i0;
    band_unit(p, u, b, g, i0);
    const int h = g * QM + hq;
    const int i = i0 + r;
    const bool row_ok = i < p.T;
    const int qp = (int)p.off + i;                // this row's position
    const int kb = band_window_start(p, i0);     // position of key column 0
    const float sink2 = p.sinks ? p.sinks[h] * LOG2E : -INFINITY;
    const uint32_t x_tm = x_tm0 + 4u * (uint32_t)(n & 1);

    fail = fail || *abort_flag || !mbar_wait(bar(BD_SFULL + X), (uint32_t)(n & 1));
    tc_fence_after();
    // admitted columns: keys max(qp - W + 1, 0) .. qp
    const int cmin = max(qp - p.window + 1, 0) - kb;
    const int cmax = qp - kb;
    // masks chunk j's scores in registers and, for pass 2, in TMEM
    auto mask16 = [&](uint32_t (&v)[16], int j) {
      const int c0 = 16 * j;
      if (__any_sync(0xffffffffu, c0 < cmin || c0 + 15 > cmax)) {
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c0 + c < cmin || c0 + c > cmax) v[c] = __float_as_uint(-INFINITY);
        tmem_st16(s_tm + c0, v);
      }
    };
    // pass 1: this half's row maximum, two chunks per TMEM round trip
    float mx = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < C::NMAX / 32; jj += 2) {
      if (jj < nh) {   // warp-uniform
        uint32_t v0[16], v1[16];
        const bool two = jj + 1 < nh;
        tmem_ld16(s_tm + 16 * (j0 + jj), v0);
        if (two) tmem_ld16(s_tm + 16 * (j0 + jj + 1), v1);
        tmem_wait_ld();
        mask16(v0, j0 + jj);
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
          m0 = max3f(m0, __uint_as_float(v0[c]), __uint_as_float(v0[c + 1]));
          m1 = max3f(m1, __uint_as_float(v0[c + 2]), __uint_as_float(v0[c + 3]));
        }
        if (two) {
          mask16(v1, j0 + jj + 1);
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            m0 = max3f(m0, __uint_as_float(v1[c]), __uint_as_float(v1[c + 1]));
            m1 = max3f(m1, __uint_as_float(v1[c + 2]), __uint_as_float(v1[c + 3]));
          }
        }
        mx = fmaxf(mx, fmaxf(m0, m1));
      }
    }
    // trade maxima with the other half of the row; all of the pipeline
    // leaves here, or none
    tmem_st1(x_tm + hf, __float_as_uint(mx));
    tmem_wait_st();
    tc_fence_before();
    if (fail) *abort_flag = 1;
    if (named_bar_or(pipe_bar, 256, fail || *abort_flag)) break;
    tc_fence_after();
    mx = fmaxf(mx, __uint_as_float(tmem_ld1(x_tm + (1 - hf))));
    tmem_wait_ld();
    // the row's maximum in log2 units, the sink included (scale > 0)
    const float mrow = fmaxf(sink2, mx * scale);
    const float neg = (mrow == -INFINITY) ? 0.f : -mrow;
    // pass 2: exp2, the partial sum, P. P of chunk j (8 bf16-pair columns)
    // goes over the first half of S chunk j's own columns, already read.
    float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
    auto exp_chunk = [&](uint32_t (&v)[16], int j) {   // scores masked in pass 1
      uint32_t pk[8];
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        float x0, x1, x2, x3;
        fma2(x0, x1, __uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]), scale, scale, neg, neg);
        fma2(x2, x3, __uint_as_float(v[2 * c + 2]), __uint_as_float(v[2 * c + 3]), scale, scale, neg, neg);
        // one pair in four on the FMA pipe (polynomial exp2), the rest on MUFU
        if ((c / 2) % 2 == 0) {
          exp2_fma2(x0, x1);
        } else {
          x0 = ex2(x0);
          x1 = ex2(x1);
        }
        x2 = ex2(x2);
        x3 = ex2(x3);
        add2(l0, l1, x0, x1);
        add2(l2, l3, x2, x3);
        pk[c] = pack_bf16(x0, x1);
        pk[c + 1] = pack_bf16(x2, x3);
      }
      tmem_st8(s_tm + 16 * j, pk);
    };
#pragma unroll
    for (int jj = 0; jj < C::NMAX / 32; jj += 2) {
      if (jj < nh) {
        uint32_t v0[16], v1[16];
        const bool two = jj + 1 < nh;
        tmem_ld16(s_tm + 16 * (j0 + jj), v0);
        if (two) tmem_ld16(s_tm + 16 * (j0 + jj + 1), v1);
        tmem_wait_ld();
        exp_chunk(v0, j0 + jj);
        if (two) exp_chunk(v1, j0 + jj + 1);
      }
    }
    const float lpart = (l0 + l1) + (l2 + l3);
    tmem_st1(x_tm + 2 + hf, __float_as_uint(lpart));
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(BD_PFULL + X));

    // the next unit's queries, while the tensor core computes this unit's O
    if (blockIdx.x + (k + 2) * G < p.n_units) rotate_unit(k + 2);

    // epilogue: O / l -> bf16 over this half of the row in the stage's Q
    // area (read by the S product, which completed before S_X was signalled)
    if (*abort_flag || !mbar_wait(bar(BD_ODONE + X), (uint32_t)(n & 1))) *abort_flag = 1;
    tc_fence_after();
    const float l = lpart + __uint_as_float(tmem_ld1(x_tm + 2 + (1 - hf))) +
                    (sink2 == -INFINITY ? 0.f : ex2(sink2 + neg));
    uint32_t o32[32];
    tmem_ld32(o_tm + 32 * hf, o32);
    tmem_wait_ld();
    const float inv_l = 1.0f / l;
    uint8_t* qrow = smem + (size_t)s * C::STAGE_BYTES + (size_t)m * C::ROWB;
#pragma unroll
    for (int c = 0; c < 32; c += 8) {
      uint4 w;
      w.x = pack_bf16(__uint_as_float(o32[c + 0]) * inv_l, __uint_as_float(o32[c + 1]) * inv_l);
      w.y = pack_bf16(__uint_as_float(o32[c + 2]) * inv_l, __uint_as_float(o32[c + 3]) * inv_l);
      w.z = pack_bf16(__uint_as_float(o32[c + 4]) * inv_l, __uint_as_float(o32[c + 5]) * inv_l);
      w.w = pack_bf16(__uint_as_float(o32[c + 6]) * inv_l, __uint_as_float(o32[c + 7]) * inv_l);
      *reinterpret_cast<uint4*>(qrow + ((((uint32_t)(32 * hf + c) >> 3) ^ swz) << 4)) = w;
    }
    if (hf == 0 && row_ok && p.lse) p.lse[((long long)b * p.n_q + h) * p.T + i] = (mrow + __log2f(l)) * LN2;
    fence_proxy_async_smem();   // the TMA store reads the staged rows through the async proxy
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(BD_EPI + X));
  }
}

template <int D>
__global__ void __launch_bounds__(544, 1)
    band_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKw,
                const __grid_constant__ CUtensorMap tmVw, const __grid_constant__ CUtensorMap tmO,
                const BandParams p) {
  using C = BandCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * BD_TMEM_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * BD_ABORT_SLOT);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BD_FULL + s), 1);
      mbar_init(bar(BD_EMPTY + s), 1);
    }
    for (int X = 0; X < 2; ++X) {
      mbar_init(bar(BD_QROT + X), 8);   // one arrival per warp
      mbar_init(bar(BD_SFULL + X), 1);
      mbar_init(bar(BD_PFULL + X), 8);
      mbar_init(bar(BD_ODONE + X), 1);
      mbar_init(bar(BD_EPI + X), 8);
      mbar_init(bar(BD_DRAIN + X), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmKw);
    tma_prefetch_desc(&tmVw);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched behind the staging kernel (the call's K/V rows) with
  // programmatic stream serialization: nothing below may read memory before
  // that launch has completed.
  griddep_wait();

  if (warp == 0) {
    // The four single-thread roles are lanes 0-3 of warp 0.
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int k = 0;
      for (;; ++k) {
        const int u = blockIdx.x + k * G;
        if (u >= p.n_units || *abort_flag) break;
        const int s = k % C::NS;
        if (k >= C::NS && !mbar_wait(bar(BD_EMPTY + s), (uint32_t)(((k / C::NS) - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        int b, g, i0;
        band_unit(p, u, b, g, i0);
        const int kb = band_window_start(p, i0);
        const uint32_t st = sbase + (uint32_t)s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar(BD_FULL + s), C::Q_BYTES + 2u * (uint32_t)p.N * C::ROWB);
        tma_load_4d(st, &tmQ, bar(BD_FULL + s), 0, g * p.q_mult, i0, b);
        // The whole window as one box of N rows (negative rows read as
        // zeros), unless it wraps around a ring: then 16-row boxes, each
        // starting on a multiple of 16 positions, so that none wraps.
        const int r0 = (p.ring_cap > 0 && kb >= 0) ? kb % p.ring_cap : kb;
        if (p.ring_cap == 0 || r0 + p.N <= p.ring_cap) {
          tma_load_4d(st + C::OFF_K, &tmKw, bar(BD_FULL + s), 0, r0, g, b);
          tma_load_4d(st + C::OFF_V, &tmVw, bar(BD_FULL + s), 0, r0, g, b);
        } else {
          for (int j = 0; j < p.N / 16; ++j) {
            const int pos = kb + 16 * j;
            const int row = pos >= 0 ? pos % p.ring_cap : pos;
            tma_load_4d(st + C::OFF_K + (uint32_t)j * 16u * C::ROWB, &tmK, bar(BD_FULL + s), 0, row, g, b);
            tma_load_4d(st + C::OFF_V + (uint32_t)j * 16u * C::ROWB, &tmV, bar(BD_FULL + s), 0, row, g, b);
          }
        }
      }
      if (*abort_flag) {
        // let every copy still in flight land before the CTA can exit
        for (int kk = (k > C::NS ? k - C::NS : 0); kk < k; ++kk)
          mbar_wait_drain(bar(BD_FULL + kk % C::NS), (uint32_t)((kk / C::NS) & 1));
      }
    }
    if (lane == 1 || lane == 2) {
      // ------------------------------------------------------------ MMA issuer of pipeline X
      const int X = lane - 1;
      const uint32_t s_col = tmem + (X ? C::S_COL1 : 0);
      const uint32_t o_col = s_col + C::O_OFF;
      const uint32_t idesc_s = idesc_bf16(128, p.N, 0, 0);
      bool ok = true;
      int n = 0;
      for (int k = X;; k += 2, ++n) {
        const int u = blockIdx.x + k * G;
        if (u >= p.n_units) break;
        const uint32_t st = sbase + (uint32_t)(k % C::NS) * C::STAGE_BYTES;
        if (!mbar_wait(bar(BD_QROT + X), (uint32_t)(n & 1))) { ok = false; break; }
        // S_X holds the previous unit's P until its O = P V has completed
        if (n > 0 && !mbar_wait(bar(BD_ODONE + X), (uint32_t)((n - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint64_t qd = smem_desc(st, 16, C::SBO, C::LAYOUT);
        const uint64_t kd = smem_desc(st + C::OFF_K, 16, C::SBO, C::LAYOUT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)   // 32 bytes per K-step inside the 128-byte swizzle row
          mma_ss(s_col, qd + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(bar(BD_SFULL + X));
        if (!mbar_wait(bar(BD_PFULL + X), (uint32_t)(n & 1))) { ok = false; break; }
        tc_fence_after();
        const uint64_t vd = smem_desc(st + C::OFF_V, C::KV_BYTES, C::SBO, C::LAYOUT);
        for (int kk = 0; kk < p.N / 16; ++kk)   // 16 keys (rows of V) per K-step; P of chunk kk at 16 kk
          mma_ts(o_col, s_col + (uint32_t)kk * 16u, vd + (uint64_t)((kk * 16 * C::ROWB) >> 4), C::IDESC_PV,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(BD_ODONE + X));
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(bar(BD_DRAIN + X));
        mbar_wait_drain(bar(BD_DRAIN + X), 0);
      }
    }
    if (lane == 3) {
      // ------------------------------------------------------------ output stores
      for (int k = 0;; ++k) {
        const int u = blockIdx.x + k * G;
        if (u >= p.n_units) break;
        const int X = k & 1, s = k % C::NS;
        if (!mbar_wait(bar(BD_EPI + X), (uint32_t)((k >> 1) & 1))) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        int b, g, i0;
        band_unit(p, u, b, g, i0);
        // rows past T are dropped by the tensor map's bounds
        tma_store_4d(&tmO, sbase + (uint32_t)s * C::STAGE_BYTES, 0, g * p.q_mult, i0, b);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(bar(BD_EMPTY + s));
      }
      bulk_wait_all();   // output stores complete before the CTA exits
    }
    __syncwarp();
  } else {
    band_softmax<D>(p, smem, bar0, tmem, abort_flag, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sa
