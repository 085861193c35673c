// Flash-style sink-augmented GQA prefill on tcgen05 tensor cores.
//
// A persistent CTA per SM walks work items; an item is two 128-row query
// tiles (A, B) of one (batch, query head), and the CTA walks the BN-key tiles
// of the cache the mask admits for them:
//
//   warp 0      TMA producer: the item's two Q tiles (already rotated, rows
//               past T read as zeros) into one of two Q buffers, then the K
//               and V tiles of the head's KV group, straight from the
//               head-major cache [B][n_kv][cap][d] (rows past offset+T read as
//               zeros through the tensor map's bounds), NS-deep ring each.
//   warps 1, 2  one thread each issues the tcgen05.mma of query tile A (warp
//               1, which also owns the TMEM allocation) or B (warp 2):
//               S_X = Q_X K^T (smem x smem, fp32 in TMEM), then
//               O_X += P_X V with P_X read from its own TMEM columns (bf16).
//               The two streams are independent: each walks every K/V tile of
//               the item, multiplies the ones its tile admits and releases the
//               others at once (the ring slots count one release from each).
//   warp 3      one thread stores each normalised output tile with a TMA
//               tile store from the item's Q buffer, where the softmax
//               warps staged it.
//   warps 4-7   softmax for tile A, warps 8-11 for tile B, one query row per
//               thread (TMEM lane = row): per key tile: read S, release it at once (so the
//               tensor core computes the next S while this one is
//               exponentiated), mask, running max in log2 units, exp2, P ->
//               TMEM, and at the end O / l -> bf16 out.
//
// TMEM (512 columns): S_A, S_B (BN each), P_A, P_B (BN/2 bf16 pairs each),
// O_A, O_B (d each); BN = 128 for d = 64, 96 for d = 96, 64 for d = 128.
//
// The softmax is seeded with the sink logit (m = sink, l = 1), so the extra
// sink column of the MoE-Xtend README ("ATTENTION STACK", sink bias) is
// folded in without ever materialising it, and dropped by construction (it
// adds to l, never to O). The O rescale is lazy: the running max only moves
// when it grows by more than 2^8, which keeps every P <= 256 and the result
// exact up to rounding. A softmax thread touches O (rescale) or P_X (next
// store) only after the previous PV_X has completed (O_DONE barrier).
//
// Key tiles are aligned to tile A's diagonal (key off+i0), so a query tile
// needs a mask only on the tiles its diagonal or band edge crosses and on a
// leading partial (negative-start) tile; band layers visit only the tiles that
// intersect [p-W+1, p] -- O(T*W) work.
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
  int sched_slot;   // which counter pair of g_prefill_sched this launch uses
  int ring_cap;     // 0: cache row = position; > 0: ring cache, row = position mod ring_cap
};

// Work counters of the dynamic item schedule, one pair per launch slot (the
// host hands a slot to one launch in flight at a time): [0] items handed out
// beyond the first gridDim.x, [1] CTAs finished. The last CTA to finish
// resets both.
constexpr int kPrefillSchedSlots = 128;
__device__ int g_prefill_sched[kPrefillSchedSlots][2];

__host__ __device__ constexpr int align32(int x) { return (x + 31) / 32 * 32; }

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                              // query rows per tile
  static constexpr int BN = (D == 64) ? 128 : (D == 96 ? 96 : 64);  // keys per tile
  static constexpr int CB = (D % 64 == 0) ? 64 : 32;          // column-block width (elements)
  static constexpr int SWZ = CB * 2;                          // bytes per block row (128 / 64)
  static constexpr int NCB = D / CB;
  static constexpr uint32_t QBLOCK = 128u * SWZ;              // column block of a Q tile
  static constexpr uint32_t Q_BYTES = 128u * D * 2;
  static constexpr uint32_t KBLOCK = (uint32_t)BN * SWZ;      // column block of a K/V tile
  static constexpr uint32_t KV_BYTES = (uint32_t)BN * D * 2;
  static constexpr int NS = (D == 64) ? 4 : (D == 96 ? 3 : 2);  // K and V ring depth
  static constexpr uint32_t LAYOUT = (SWZ == 128) ? 2u : 4u;
  static constexpr uint32_t SBO = 8u * SWZ;                   // 8-row core-matrix group stride
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0, S_COL1 = BN;
  static constexpr int P_COL0 = 2 * BN, P_COL1 = 2 * BN + align32(BN / 2);
  static constexpr int O_COL0 = align32(P_COL1 + BN / 2), O_COL1 = O_COL0 + D;
  static_assert(O_COL1 + D <= TMEM_COLS, "TMEM plan exceeds 512 columns");
  static_assert(KBLOCK % 1024 == 0 && QBLOCK % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static constexpr int NUM_THREADS = 384;
  // smem: Q[2 buffers][2 tiles] | K[NS] | V[NS] | barriers
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = 4 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NS * KV_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
  static constexpr uint32_t IDESC_QK = idesc_bf16(128, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 0, 1);
};

// Barrier slots (8 bytes each) at OFF_BAR. [2] = one per Q buffer or per
// query tile X; [NS] = one per K/V ring slot.
enum : int {
  BAR_QFULL = 0,    // [2 buffers] producer (TMA) -> MMA: an item's Q tiles landed
  BAR_QEMPTY = 2,   // [2 buffers] count 4: MMA A and B (last S product read the
                    // tiles) and the two output stores (which stage O in them)
  BAR_SFULL = 4,    // [2 tiles] MMA -> softmax: S_X computed
  BAR_SFREE = 6,    // [2] softmax -> MMA: S_X read into registers
  BAR_PFULL = 8,    // [2] softmax -> MMA: P_X stored (and O_X rescaled)
  BAR_ODONE = 10,   // [2] MMA -> softmax: PV_X completed
  BAR_OFREE = 12,   // [2] softmax -> MMA: the item's epilogue has read O_X
  BAR_DRAIN = 14,   // [2] per MMA issuer, on abort
  BAR_KFULL = 16,   // [NS <= 4]
  BAR_KEMPTY = 20,  // [NS] count 2: MMA A and MMA B
  BAR_VFULL = 24,   // [NS]
  BAR_VEMPTY = 28,  // [NS] count 2
  BAR_TMEM_SLOT = 32,
  BAR_ABORT_SLOT = 33,
  BAR_IFULL = 38,   // [4] producer -> every role: item descriptor k published in ring slot k & 3
  BAR_IEMPTY = 42,  // [4] count 11 (MMA A, MMA B, store thread, 8 softmax warps): read
  BAR_IRING = 46,   // int {item, pair, h, b}[4] then float sink[4] (slots 46-55)
  BAR_EPI = 34,     // [2 X][2 Q buffers] softmax X warps -> the store thread: O rows
                    // staged in Q buffer b (one barrier per buffer, so a pipeline
                    // running an item ahead cannot complete a phase twice)
};

// Work items are (query-tile pair, query head, sequence), numbered heaviest
// pair first. CTA c starts with item c; every further item comes from an
// atomic counter (dynamic schedule: an SM that finishes early takes more, so
// neither the uneven item sizes nor uneven SM speeds leave a tail). The
// producer thread fetches the ids and publishes each, with its sink logit, in
// a 4-slot shared-memory ring that every role reads in the same order.
struct ItemSchedule {
  int G, n_items, per_pair, n_pairs, n_q;
  // The two pipelines trade row tiles on every other item of a CTA
  // (pipeline X takes row tile X ^ 1): the upper tile of a causal pair has one
  // key tile more, and alternating it keeps both pipelines equally loaded.
  __device__ __forceinline__ static int swap(int k) { return k & 1; }
  __device__ __forceinline__ void coords(int item, int& pair, int& h, int& b) const {
    const int rank = item / per_pair, rem = item % per_pair;
    pair = n_pairs - 1 - rank;
    h = rem % n_q;
    b = rem / n_q;
  }
};

// Positions (offset + row) fit in 32 bits: the cache capacity and every
// offset are below 2^31.
__device__ __forceinline__ int floordiv(int a, int b) {  // b > 0
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}

// Key-tile geometry of one CTA: tile t covers keys [base + BN t, base + BN t + BN).
// For query tile X (rows i0 + 128 X .. + 127, positions p = off + row):
//   active tiles  [a_lo[X], a_hi[X]): the tile meets the admitted keys of some row;
//   full tiles    [f_lo[X], f_hi[X]): every key of the tile is admitted for all
//                 128 rows (0 <= key <= p, and key > p - W on band layers), so
//                 no mask is applied there.
template <int BN>
struct TileGeom {
  int off;
  int T, window;
  int i0;          // first query row of tile A
  int base;        // first key of key tile 0
  int ntiles;
  int a_lo[2], a_hi[2], f_lo[2], f_hi[2];
  __device__ __forceinline__ bool valid(int X) const { return i0 + 128 * X < T; }
  __device__ __forceinline__ int lo(int X) const {
    const int p0 = off + i0 + 128 * X;
    return window > 0 ? (p0 - window + 1 > 0 ? p0 - window + 1 : 0) : 0;
  }
  __device__ __forceinline__ int hi(int X) const {  // exclusive
    const int last = min(T, i0 + 128 * X + 128);
    return off + last;
  }
  __device__ __forceinline__ bool active(int X, int t) const { return t >= a_lo[X] && t < a_hi[X]; }
  __device__ __forceinline__ bool full(int X, int t) const { return t >= f_lo[X] && t < f_hi[X]; }
};

template <int BN>
__device__ __forceinline__ TileGeom<BN> make_geom(const PrefillParams& p, int pair) {
  TileGeom<BN> g;
  g.off = (int)p.off;
  g.T = p.T;
  g.window = p.window;
  g.i0 = pair * 256;
  const int diag = g.off + g.i0;
  const int loA = g.lo(0);
  if (p.ring_cap > 0) {
    // ring cache: key tiles start at multiples of BN, so none wraps around
    g.base = floordiv(loA, BN) * BN;
  } else {
    // key tiles aligned to tile A's diagonal: one masked tile per query tile
    const int nb = (diag - loA + BN - 1) / BN;
    g.base = diag - BN * nb;
  }
  const int hi = g.off + min(p.T, g.i0 + 256);
  g.ntiles = (hi - g.base + BN - 1) / BN;
#pragma unroll
  for (int X = 0; X < 2; ++X) {
    if (!g.valid(X)) {
      g.a_lo[X] = g.a_hi[X] = g.f_lo[X] = g.f_hi[X] = 0;
      continue;
    }
    // active: klo < hi(X) and klo + BN > lo(X)
    const int alo = floordiv(g.lo(X) - g.base, BN);
    const int ahi = floordiv(g.hi(X) - g.base + BN - 1, BN);
    g.a_lo[X] = alo < 0 ? 0 : alo;
    g.a_hi[X] = ahi > g.ntiles ? g.ntiles : ahi;
    // full: klo >= 0, klo + BN - 1 <= p0, and (band) klo > p0 + 127 - W
    const int p0 = g.off + g.i0 + 128 * X;
    int flo = floordiv(-g.base + BN - 1, BN);
    if (p.window > 0) {
      const int w = floordiv(p0 + 127 - p.window - g.base, BN) + 1;
      if (w > flo) flo = w;
    }
    const int fhi = floordiv(p0 - BN + 1 - g.base, BN) + 1;
    g.f_lo[X] = flo < g.a_lo[X] ? g.a_lo[X] : (flo > g.a_hi[X] ? g.a_hi[X] : flo);
    g.f_hi[X] = fhi > g.a_hi[X] ? g.a_hi[X] : (fhi < g.f_lo[X] ? g.f_lo[X] : fhi);
  }
  return g;
}

// MMA issue helpers (one thread). Descriptors are built once per CTA and
// advanced by compile-time offsets of their start-address field (16-byte
// units; every operand stays below 256 KB of shared memory, so the 14-bit
// field never carries).
// S_X = Q_X K_t^T over d/16 K-steps.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint64_t qdesc, uint64_t kdesc) {
  using C = PrefillCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t cb = kk * 16 / C::CB, cin = (kk * 16 % C::CB) * 2;
    mma_ss(s_tmem, qdesc + ((cb * C::QBLOCK + cin) >> 4), kdesc + ((cb * C::KBLOCK + cin) >> 4),
           C::IDESC_QK, kk > 0 ? 1u : 0u);
  }
}
// O_X (+)= P_X V_t over BN/16 K-steps; P_X is bf16 in TMEM.
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t vdesc,
                                         bool accumulate) {
  using C = PrefillCfg<D>;
#pragma unroll
  for (int kk = 0; kk < C::BN / 16; ++kk)
    mma_ts(o_tmem, p_tmem + kk * 8, vdesc + ((kk * 16 * C::SWZ) >> 4), C::IDESC_PV,
           (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const PrefillParams p) {
  using C = PrefillCfg<D>;
  constexpr int BN = C::BN;
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
  ItemSchedule sched;
  sched.G = gridDim.x;
  sched.per_pair = p.n_q * p.B;
  sched.n_pairs = p.n_pairs;
  sched.n_items = p.n_pairs * sched.per_pair;
  sched.n_q = p.n_q;
  volatile int4* ring_item = reinterpret_cast<volatile int4*>(smem + C::OFF_BAR + 8 * BAR_IRING);
  volatile float* ring_sink = reinterpret_cast<volatile float*>(smem + C::OFF_BAR + 8 * BAR_IRING + 64);
  // Read item k of this CTA from the ring (all roles, in order): its id,
  // coordinates and sink; `elected`: whether this thread arrives on the
  // slot's release barrier for its group. Returns n_items (no more work) on a
  // timed-out wait.
  auto fetch = [&](int k, bool elected, int& pair, int& h, int& b, float& sink) -> int {
    const int sl = k & 3;
    if (!mbar_wait(bar(BAR_IFULL + sl), (uint32_t)((k >> 2) & 1))) {
      *abort_flag = 1;
      return sched.n_items;
    }
    const int it = ring_item[sl].x;
    pair = ring_item[sl].y;
    h = ring_item[sl].z;
    b = ring_item[sl].w;
    sink = ring_sink[sl];
    __syncwarp(__activemask());
    if (elected) mbar_arrive(bar(BAR_IEMPTY + sl));
    return it;
  };

  if (threadIdx.x == 0) {
    for (int X = 0; X < 2; ++X) {
      mbar_init(bar(BAR_QFULL + X), 1);
      mbar_init(bar(BAR_QEMPTY + X), 4);
      mbar_init(bar(BAR_EPI + 2 * X), 4);   // one arrival per warp
      mbar_init(bar(BAR_EPI + 2 * X + 1), 4);
      mbar_init(bar(BAR_SFULL + X), 1);
      mbar_init(bar(BAR_SFREE + X), 4);   // one arrival per warp
      mbar_init(bar(BAR_PFULL + X), 4);   // one arrival per warp
      mbar_init(bar(BAR_ODONE + X), 1);
      mbar_init(bar(BAR_OFREE + X), 4);   // one arrival per warp
      mbar_init(bar(BAR_DRAIN + X), 1);
    }
    for (int sl = 0; sl < 4; ++sl) {
      mbar_init(bar(BAR_IFULL + sl), 1);
      mbar_init(bar(BAR_IEMPTY + sl), 11);
    }
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_KEMPTY + s), 2);
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_VEMPTY + s), 2);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched behind the staging kernel with programmatic stream
  // serialization: the set-up above overlaps its tail; nothing below may read
  // memory before it has completed (the staged queries, the appended rows).
  griddep_wait();

  if (warp < 4) {
    // Warpgroup 0: producer (warp 0), MMA issuers (warps 1, 2). It gives
    // registers to the two softmax warpgroups: 128*72 + 256*216 = 384*168,
    // the launch allocation.
    regs_dec<72>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ producer
      int gt = 0;  // K/V tiles issued so far (ring position)
      int j = 0;   // Q loads issued so far
      int* ctr = &g_prefill_sched[p.sched_slot][0];
      int next = blockIdx.x;   // the first item; later ones from the counter
      for (int k = 0; !*abort_flag; ++k) {
        const int sl = k & 3;
        if (k >= 4 && !mbar_wait(bar(BAR_IEMPTY + sl), (uint32_t)(((k >> 2) - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        const int item = next < sched.n_items ? next : sched.n_items;
        int pair = 0, h = 0, b = 0;
        float sink = -INFINITY;
        if (item < sched.n_items) {
          next = sched.G + atomicAdd(ctr, 1);   // the following item, fetched one ahead
          sched.coords(item, pair, h, b);
          if (p.sinks) sink = p.sinks[h];
        }
        ring_item[sl].x = item;
        ring_item[sl].y = pair;
        ring_item[sl].z = h;
        ring_item[sl].w = b;
        ring_sink[sl] = sink;
        mbar_arrive(bar(BAR_IFULL + sl));   // release: the ring entry is visible to acquirers
        if (item >= sched.n_items) break;
        const int rr = k;
        const int g = h / p.q_mult;
        const TileGeom<BN> geo = make_geom<BN>(p, pair);
        const int qb = j & 1;
        if (j >= 2 && !mbar_wait(bar(BAR_QEMPTY + qb), (uint32_t)(((j >> 1) - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        // pipeline X takes row tile X ^ sw (see ItemSchedule::swap)
        const int sw = ItemSchedule::swap(rr);
        const int nq = geo.valid(1) ? 2 : 1;
        mbar_arrive_expect_tx(bar(BAR_QFULL + qb), (uint32_t)nq * C::Q_BYTES);
        for (int X = 0; X < 2; ++X) {
          const int rt = X ^ sw;
          if (!geo.valid(rt)) continue;
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_4d(sbase + C::OFF_Q + (2 * qb + X) * C::Q_BYTES + cb * C::QBLOCK, &tmQ,
                        bar(BAR_QFULL + qb), cb * C::CB, geo.i0 + 128 * rt, h, b);
        }
        ++j;
        for (int t = 0; t < geo.ntiles; ++t, ++gt) {
          const int s = gt % C::NS;
          const uint32_t ph = (uint32_t)((gt / C::NS) & 1);
          const int kpos = geo.base + BN * t;
          const int krow = p.ring_cap > 0 ? kpos % p.ring_cap : kpos;
          if (!mbar_wait(bar(BAR_KEMPTY + s), ph ^ 1)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(bar(BAR_KFULL + s), C::KV_BYTES);
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_4d(sbase + C::OFF_K + s * C::KV_BYTES + cb * C::KBLOCK, &tmK, bar(BAR_KFULL + s),
                        cb * C::CB, krow, g, b);
          if (!mbar_wait(bar(BAR_VEMPTY + s), ph ^ 1)) {
            *abort_flag = 1;
            // K(gt) is in flight, V(gt) is not
            mbar_wait_drain(bar(BAR_KFULL + s), ph);
            break;
          }
          mbar_arrive_expect_tx(bar(BAR_VFULL + s), C::KV_BYTES);
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_4d(sbase + C::OFF_V + s * C::KV_BYTES + cb * C::KBLOCK, &tmV, bar(BAR_VFULL + s),
                        cb * C::CB, krow, g, b);
        }
      }
      if (*abort_flag) {
        // Let every copy still in flight land before the CTA can exit.
        for (int u = (gt > C::NS ? gt - C::NS : 0); u < gt; ++u) {
          mbar_wait_drain(bar(BAR_KFULL + u % C::NS), (uint32_t)((u / C::NS) & 1));
          mbar_wait_drain(bar(BAR_VFULL + u % C::NS), (uint32_t)((u / C::NS) & 1));
        }
        for (int u = (j > 2 ? j - 2 : 0); u < j; ++u)
          mbar_wait_drain(bar(BAR_QFULL + (u & 1)), (uint32_t)((u >> 1) & 1));
      }
    } else if (warp == 3 && lane == 0) {
      // ------------------------------------------------------------ output stores
      // Per item and query tile: once the softmax warps have staged the
      // normalised output tile in the item's Q buffer (BAR_EPI), one TMA
      // tile store; the Q buffer is released to the producer once the stores
      // have read it.
      int j = 0;
      int nepi[2][2] = {{0, 0}, {0, 0}};   // phases of BAR_EPI [X][buffer]
      bool ok = true;
      for (int rr = 0; ok; ++rr) {
        float sink_unused;
        int pair, h, b;
        const int item = fetch(rr, true, pair, h, b, sink_unused);
        if (item >= sched.n_items) break;
        const TileGeom<BN> geo = make_geom<BN>(p, pair);
        const int sw = ItemSchedule::swap(rr);
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          const int rt = X ^ sw;
          if (!geo.valid(rt)) continue;
          const int qb = j & 1;
          if (!mbar_wait(bar(BAR_EPI + 2 * X + qb), (uint32_t)(nepi[X][qb] & 1))) { ok = false; *abort_flag = 1; break; }
          ++nepi[X][qb];
          if (*abort_flag) { ok = false; break; }
          const uint32_t stage = sbase + C::OFF_Q + (2 * (j & 1) + X) * C::Q_BYTES;
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_store_4d(&tmO, stage + cb * C::QBLOCK, cb * C::CB, geo.i0 + 128 * rt, h, b);
          bulk_commit();
        }
        if (!ok) break;
        bulk_wait_read_all();
        mbar_arrive(bar(BAR_QEMPTY + (j & 1)));   // both staged tiles have been read
        mbar_arrive(bar(BAR_QEMPTY + (j & 1)));
        ++j;
      }
      bulk_wait_all();   // output stores complete before the CTA exits
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ------------------------------------------------------------ MMA issuer of tile X
      // Per key tile t: S_X(t) as soon as the softmax released the previous
      // S_X; then O_X += P_X(t-1) V(t-1). Tiles outside X's range are only
      // released. Every wait is bounded; a failed one aborts the CTA.
      const int X = warp - 1;
      const uint32_t s_col = tmem + (X ? C::S_COL1 : C::S_COL0);
      const uint32_t p_col = tmem + (X ? C::P_COL1 : C::P_COL0);
      const uint32_t o_col = tmem + (X ? C::O_COL1 : C::O_COL0);
      const uint32_t b_sfull = bar(BAR_SFULL + X), b_sfree = bar(BAR_SFREE + X);
      const uint32_t b_pfull = bar(BAR_PFULL + X), b_odone = bar(BAR_ODONE + X);
      const uint32_t b_ofree = bar(BAR_OFREE + X);
      bool ok = true;
      const uint64_t kd0 = smem_desc(sbase + C::OFF_K, 16, C::SBO, C::LAYOUT);
      const uint64_t vd0 = smem_desc(sbase + C::OFF_V, C::KBLOCK, C::SBO, C::LAYOUT);
      int nS = 0, nP = 0;  // cumulative S products / PV products of this tile
      int gt = 0;          // ring position of K(0) of the current item
      int j = 0;           // items done by this CTA
      for (int rr = 0; ok; ++rr) {
        float sink_unused;
        int pair, h, b;
        const int item = fetch(rr, true, pair, h, b, sink_unused);
        if (item >= sched.n_items) break;
        const TileGeom<BN> geo = make_geom<BN>(p, pair);
        const int qb = j & 1;
        if (!mbar_wait(bar(BAR_QFULL + qb), (uint32_t)((j >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint64_t qd = smem_desc(sbase + C::OFF_Q + (2 * qb + X) * C::Q_BYTES, 16, C::SBO, C::LAYOUT);
        const int rt = X ^ ItemSchedule::swap(rr);   // row tile of this pipeline
        const int lo = rt ? geo.a_lo[1] : geo.a_lo[0], hi = rt ? geo.a_hi[1] : geo.a_hi[0];
        if (hi <= lo) mbar_arrive(bar(BAR_QEMPTY + qb));   // this tile reads no Q
        bool first = true;                                  // no PV of this item issued yet
        for (int t = 0; t <= geo.ntiles; ++t) {
          if (t < geo.ntiles) {
            const int u = gt + t;
            const int ks = u % C::NS;
            if (!mbar_wait(bar(BAR_KFULL + ks), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
            if (t >= lo && t < hi) {
              if (nS > 0 && !mbar_wait(b_sfree, (uint32_t)((nS - 1) & 1))) { ok = false; break; }
              tc_fence_after();
              issue_qk<D>(s_col, qd, kd0 + ((uint32_t)(ks * C::KV_BYTES) >> 4));
              mma_commit(b_sfull);
              ++nS;
              if (t == hi - 1) mma_commit(bar(BAR_QEMPTY + qb));   // last read of this Q tile
              mma_commit(bar(BAR_KEMPTY + ks));
            } else {
              mbar_arrive(bar(BAR_KEMPTY + ks));
            }
          }
          if (t > 0) {
            const int u = gt + t - 1;
            const int vs = u % C::NS;
            if (!mbar_wait(bar(BAR_VFULL + vs), (uint32_t)((u / C::NS) & 1))) { ok = false; break; }
            if (t - 1 >= lo && t - 1 < hi) {
              if (first && j > 0 && !mbar_wait(b_ofree, (uint32_t)((j - 1) & 1))) { ok = false; break; }
              if (!mbar_wait(b_pfull, (uint32_t)(nP & 1))) { ok = false; break; }
              tc_fence_after();
              issue_pv<D>(o_col, p_col, vd0 + ((uint32_t)(vs * C::KV_BYTES) >> 4), !first);
              mma_commit(b_odone);
              ++nP;
              first = false;
              mma_commit(bar(BAR_VEMPTY + vs));
            } else {
              mbar_arrive(bar(BAR_VEMPTY + vs));
            }
          }
          if (*abort_flag) { ok = false; break; }
        }
        gt += geo.ntiles;
        ++j;
      }
      if (!ok) {
        *abort_flag = 1;
        // Drain this issuer's tensor-core work before anything is released.
        mma_commit(bar(BAR_DRAIN + X));
        mbar_wait_drain(bar(BAR_DRAIN + X), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    regs_inc<216>();
    const int X = (warp - 4) >> 2;
    const int quarter = warp & 3;               // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;          // row within the query tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + (X ? C::S_COL1 : C::S_COL0);
    const uint32_t p_tm = tmem + lane_base + (X ? C::P_COL1 : C::P_COL0);
    const uint32_t o_tm = tmem + lane_base + (X ? C::O_COL1 : C::O_COL0);
    const float LOG2E = 1.4426950408889634f;
    const float scale = p.scale_log2;
    int ntot = 0;   // cumulative key tiles of this query tile slot (S / P / O-done phases)
    int j = 0;      // items of this CTA so far (Q buffer j & 1 stages this item's output)
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
      float sink_raw;
      int pair, h, b;
      const int item = fetch(rr, lane == 0, pair, h, b, sink_raw);
      if (item >= sched.n_items) break;
      const TileGeom<BN> geo = make_geom<BN>(p, pair);
      const int rt = X ^ ItemSchedule::swap(rr);   // row tile of this pipeline
      const int i = geo.i0 + 128 * rt + r;      // query row within the call
      const bool row_ok = i < p.T;
      const long long pos = p.off + i;
      if (geo.valid(rt)) {
        const float sink2 = sink_raw * LOG2E;   // -inf without sinks
        float m = sink2;                              // running max (log2 units)
        float l = (sink2 == -INFINITY) ? 0.f : 1.f;   // running sum, sink included
        int n = 0;                                    // key tiles of this item
        const int t_lo = rt ? geo.a_lo[1] : geo.a_lo[0], t_hi = rt ? geo.a_hi[1] : geo.a_hi[0];
        const int full_lo = rt ? geo.f_lo[1] : geo.f_lo[0], full_hi = rt ? geo.f_hi[1] : geo.f_hi[0];
        for (int t = t_lo; t < t_hi; ++t) {
          if (!mbar_wait(bar(BAR_SFULL + X), (uint32_t)(ntot & 1))) { ok = false; *abort_flag = 1; break; }
          tc_fence_after();
          uint32_t sr[BN];
#pragma unroll
          for (int c0 = 0; c0 < BN; c0 += 32)
            tmem_ld32(s_tm + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[c0]));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_SFREE + X));   // the tensor core may overwrite S_X now
          if (t < full_lo || t >= full_hi) {
            // Admitted columns c (key klo + c) satisfy cmin <= c <= cmax. A
            // tile needs the upper bound where it crosses the diagonal of
            // some row and the lower one where it reaches below the band (or
            // below key 0) of some row; each side is one compare + select
            // per column, skipped when no row of the tile needs it.
            // Positions fit in 32 bits (cap < 2^31).
            const int klo = geo.base + BN * t;
            const int p0 = (int)p.off + geo.i0 + 128 * rt;   // position of row 0
            const int ipos = (int)pos;
            if (klo + BN - 1 > p0) {
              const int cmax = min(max(ipos - klo, -1), BN);
#pragma unroll
              for (int c = 0; c < BN; ++c)
                if (c > cmax) sr[c] = __float_as_uint(-INFINITY);
            }
            const int lo_last = p.window > 0 ? max(p0 + 128 - p.window, 0) : 0;   // lowest key of row 127
            if (klo < lo_last) {
              const int lo_k = p.window > 0 ? max(ipos - p.window + 1, 0) : 0;
              const int cmin = min(max(lo_k - klo, 0), BN);
#pragma unroll
              for (int c = 0; c < BN; ++c)
                if (c < cmin) sr[c] = __float_as_uint(-INFINITY);
            }
          }
          // raw row max (scale > 0, so max(s * scale) = scale * max(s))
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < BN; c += 8) {
            m0 = max3f(m0, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
            m1 = max3f(m1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
            m2 = max3f(m2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
            m3 = max3f(m3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
          }
          const float mx = fmaxf(max3f(m0, m1, m2), m3) * scale;
          const float m_new = fmaxf(m, mx);
          const bool need = m_new > m + 8.0f;
          // O_X is rescaled by f later, once the previous PV_X has landed.
          const bool rescale = __any_sync(0xffffffffu, need) && n > 0;
          float f = 1.0f;
          if (need) {
            f = ex2(m - m_new);
            l *= f;
            m = m_new;
          }
          const float neg = (m == -INFINITY) ? 0.f : -m;
          uint32_t pk[BN / 2];
          float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
          for (int c = 0; c < BN / 2; c += 2) {
            float x0, x1, x2, x3;
            fma2(x0, x1, __uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]), scale, scale, neg, neg);
            fma2(x2, x3, __uint_as_float(sr[2 * c + 2]), __uint_as_float(sr[2 * c + 3]), scale, scale, neg, neg);
            // One pair in four goes to the FMA pipe (polynomial exp2), the
            // rest to the MUFU unit: the two run side by side.
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
          l += (l0 + l1) + (l2 + l3);
          // O_X and P_X are read by the previous PV_X until it completes.
          if (ntot > 0) {
            if (!mbar_wait(bar(BAR_ODONE + X), (uint32_t)((ntot - 1) & 1))) { ok = false; *abort_flag = 1; break; }
            tc_fence_after();
          }
          if (rescale) {
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o32[32];
              tmem_ld32(o_tm + c0, o32);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                float a0 = __uint_as_float(o32[c]), a1 = __uint_as_float(o32[c + 1]);
                mul2(a0, a1, f, f);
                o32[c] = __float_as_uint(a0);
                o32[c + 1] = __float_as_uint(a1);
              }
              tmem_st32(o_tm + c0, o32);
            }
          }
#pragma unroll
          for (int c0 = 0; c0 + 32 <= BN / 2; c0 += 32)
            tmem_st32(p_tm + c0, *reinterpret_cast<uint32_t(*)[32]>(&pk[c0]));
          if constexpr ((BN / 2) % 32 == 16) tmem_st16(p_tm + (BN / 2 - 16), &pk[BN / 2 - 16]);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_PFULL + X));
          ++n;
          ++ntot;
          if (*abort_flag) { ok = false; break; }
        }
        // Epilogue, once the item's last PV_X has landed: O / l -> bf16 into
        // this pipeline's Q tile of the item (its last S product has been
        // read, so the tile is free), then one TMA store of the 128 x d tile
        // (rows past T are dropped by the tensor map's bounds).
        uint8_t* stage = smem + C::OFF_Q + (2 * (j & 1) + X) * C::Q_BYTES;
        if (ok && n > 0 && mbar_wait(bar(BAR_ODONE + X), (uint32_t)((ntot - 1) & 1)) && !*abort_flag) {
          tc_fence_after();
          const float inv_l = 1.0f / l;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o32[32];
            tmem_ld32(o_tm + c0, o32);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(o32[c + 0]) * inv_l, __uint_as_float(o32[c + 1]) * inv_l);
              v.y = pack_bf16(__uint_as_float(o32[c + 2]) * inv_l, __uint_as_float(o32[c + 3]) * inv_l);
              v.z = pack_bf16(__uint_as_float(o32[c + 4]) * inv_l, __uint_as_float(o32[c + 5]) * inv_l);
              v.w = pack_bf16(__uint_as_float(o32[c + 6]) * inv_l, __uint_as_float(o32[c + 7]) * inv_l);
              *reinterpret_cast<uint4*>(stage + swz_off<C::CB>(r, c0 + c, C::QBLOCK)) = v;
            }
          }
          if (row_ok && p.lse) {
            const float LN2 = 0.6931471805599453f;
            p.lse[((long long)b * p.n_q + h) * p.T + i] = (m + __log2f(l)) * LN2;
          }
        } else if (!ok || *abort_flag) {
          ok = false;
          *abort_flag = 1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_EPI + 2 * X + (j & 1)));   // warp 3 stores the tile
      }
      ++j;
      // O_X is free for the next item's first PV.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_OFREE + X));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) {
    // Every producer of the grid has fetched its last id once all CTAs got
    // here, so the last one can reset the counters for the next launch.
    __threadfence();
    if (atomicAdd(&g_prefill_sched[p.sched_slot][1], 1) == (int)gridDim.x - 1) {
      g_prefill_sched[p.sched_slot][0] = 0;
      g_prefill_sched[p.sched_slot][1] = 0;
      __threadfence();
    }
  }
}

}  // namespace sa
