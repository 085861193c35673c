// One-token sink-augmented GQA decode, split across SMs.
//
// The work is reading the KV cache once: for each (sequence b, KV head g)
// the rows [lo, off) are cut into stages of R rows, streamed by S CTAs
// (grid n_kv x S x B): each CTA first takes a contiguous run of stages of its
// own (about half of its share, prefetched into L2 before the kernel ahead
// of it has finished), then asks a per-(b, g) counter for one more stage at
// a time until none is left, so CTAs that happen to stream faster do more
// and all of them finish together. Inside a CTA one producer warp streams 128-row K and V
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
// CTA writes its partial to the workspace as one record and the last CTA of
// (b, g) to finish (atomic ticket, no spinning) brings all S records into its
// idle K/V ring with one bulk copy and merges them with the sink:
// M = max(max_s m_s, sink), l = sum_s e^{m_s-M} l_s + e^{sink-M},
// out = sum_s e^{m_s-M} O_s / l.
//
// FP8 caches (decode_kernel<D, true>) store e4m3 codes plus one fp32 scale
// per row (fp8.cuh). Their stages carry R codes rows of K and of V and the
// 2R row scales; a consumer converts codes to f16 in registers (exact), so
// K enters S^T = K Q^T unscaled and each score is multiplied by its row's K
// scale afterwards, while each probability is multiplied by its row's V
// scale before it becomes the f16 operand of O^T = V^T P^T. To keep those
// f16 operands in range, Q is taken in f16 after a per-head power-of-two
// scaling (undone in the score scale), and P*scale_v is taken relative to a
// per-warp power of two that only grows (undone when the warp's partial is
// written). Rows of a sub-tile are visited in a permuted order chosen so
// that the byte-granular shared-memory reads of V hit distinct banks.
#pragma once

#include <type_traits>

#include "fp8.cuh"
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
  long long n_blocks;  // stages of R rows from lo to off (each (b, g) streams all of them)
  int static_stages;   // split s first takes stages [s F, s F + F); stages from S F on are
                       // handed out one at a time by ws_grab[b][g] to whichever CTA asks first
  float* cks;       // FP8 caches: row scales [B][n_kv][cap] of K and of V
  float* cvs;
  int S;
  int pf_stages;    // stages each CTA prefetches into L2 before waiting for its predecessor
  float scale_log2;
  int rope;
  float* ws_rec;   // [B][n_kv][S] records of rec_floats: O [q_mult][D], m [q_mult], l [q_mult]
  int rec_floats;  // q_mult * D + (2 q_mult rounded up to a multiple of 4): 16-byte records
  int* ws_cnt;     // [B][n_kv] split tickets
  int* ws_grab;    // [B][n_kv] next dynamic stage (both end every call at zero)
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
  static constexpr uint32_t RING_BYTES = 2 * NS * STAGE_BYTES;   // K and V stages
  static constexpr uint32_t OFF_BAR = OFF_XV + XTILE;
  // after the 2 NS ring barriers: the merge barrier, two flags, the sinks
  static constexpr uint32_t OFF_MBAR = OFF_BAR + 8 * (2 * NS);
  static constexpr uint32_t OFF_FLAG = OFF_MBAR + 8;
  static constexpr uint32_t OFF_SINK = OFF_FLAG + 16;
  static constexpr uint32_t OFF_SROW = OFF_SINK + 32;   // [NS] first cache position of each stage
  static constexpr uint32_t SMEM_BYTES = OFF_SROW + 8 * NS + 1024;
  static constexpr int BLKCOLS = CB;                    // tensor-map columns per column block
  static constexpr uint32_t STAGE_TX = 2 * STAGE_BYTES;  // bytes one stage's TMA loads bring
  static constexpr int RW = 16;                         // rows per consumer warp per stage
  static constexpr int NBOX = 1;                        // 128-row TMA boxes per stage
};

// FP8 caches: codes rows of D bytes, stored as column blocks of ROWB bytes
// (one swizzle span: 64 B for d = 64, 128 B for d = 128, 3 x 32 B for d = 96),
// with the stage's 128 K and 128 V row scales beside them.
template <int D>
struct DecodeF8Cfg {
  static constexpr int NCW = 8;
  // rows per consumer warp and stage: two 16-row sub-tiles (their dependent
  // chains interleave) where shared memory allows; a stage is loaded as
  // 128-row TMA boxes, each starting on a multiple of 128 positions, so no
  // box wraps a ring
  static constexpr int RW = (D == 128) ? 16 : 32;
  static constexpr int R = RW * NCW;
  static constexpr int NBOX = R / 128;
  static constexpr int ROWB = (D == 96) ? 32 : D;
  static constexpr int NCB = D / ROWB;
  static constexpr int BLKCOLS = ROWB;
  static constexpr uint32_t BLOCK_BYTES = R * ROWB;
  static constexpr uint32_t STAGE_BYTES = R * D;        // K (or V) codes of one stage
  // about as many bytes in flight per CTA as the bf16 kernel keeps
  static constexpr int NS = (D == 96) ? 2 : 3;
  static constexpr uint32_t STAGE_TX = 2 * STAGE_BYTES + 2 * R * 4;
  static constexpr uint32_t XBLOCK = 16 * ROWB;
  static constexpr uint32_t XTILE = 16 * D;
  static constexpr int NUM_THREADS = 32 * (NCW + 1);
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = NS * STAGE_BYTES;
  static constexpr uint32_t OFF_KS = 2 * NS * STAGE_BYTES;   // [NS][R] fp32
  static constexpr uint32_t OFF_VS = OFF_KS + NS * R * 4;
  static constexpr uint32_t OFF_XK = OFF_VS + NS * R * 4;
  static constexpr uint32_t OFF_XV = OFF_XK + XTILE;
  static constexpr uint32_t OFF_XS = OFF_XV + XTILE;         // [2][16] fp32: new-row scales
  static_assert(RW % 16 == 0 && R % 128 == 0, "stages are whole 128-row boxes of 16-row sub-tiles");
  static constexpr uint32_t OFF_RED = OFF_K;
  static constexpr uint32_t RED_WARP = (16 + 8 * D) * 4;
  static_assert(NCW * RED_WARP <= 2 * NS * STAGE_BYTES, "warp partials must fit in the ring");
  static_assert(OFF_XK % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr uint32_t RING_BYTES = 2 * NS * STAGE_BYTES;   // K and V codes
  static constexpr uint32_t OFF_BAR = OFF_XS + 128;
  static constexpr uint32_t OFF_MBAR = OFF_BAR + 8 * (2 * NS);
  static constexpr uint32_t OFF_FLAG = OFF_MBAR + 8;
  static constexpr uint32_t OFF_SINK = OFF_FLAG + 16;
  static constexpr uint32_t OFF_SROW = OFF_SINK + 32;   // [NS] first cache position of each stage
  static constexpr uint32_t SMEM_BYTES = OFF_SROW + 8 * NS + 1024;
};

template <int D, bool F8>
using DecodeCfgT = typename std::conditional<F8, DecodeF8Cfg<D>, DecodeCfg<D>>::type;

// Physical row (within a 16-row sub-tile) of logical key L of the FP8
// consumer: logical keys {2c, 2c+1, 2c+8, 2c+9} of lane group c must sit in
// rows whose swizzled V words fall in distinct banks.
template <int D>
__device__ __forceinline__ int f8_row(int L) {
  const int l = L & 7;
  const int r = (D == 64) ? (2 * (l & 3) + (l >> 2)) : (D == 96 ? ((l >> 1) + 4 * (l & 1)) : l);
  return (L & 8) | r;
}

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
    // the accumulators move only when some head's maximum grew (alpha < 1)
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        o[md][e] *= alpha;
        o[md][2 + e] *= alpha;
      }
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

// Shared-memory offsets (from a stage's K or V base) that the FP8 consumer
// lane reads for a warp whose sub-tiles start at tile row row0, in 32-byte
// column group 0 (grp_addr gives the others): ko[u] its ldmatrix row of
// sub-tile u, vo[u][i] the V rows of logical keys 2cq, 2cq+1, 2cq+8, 2cq+9.
template <int D, int NSUB>
__device__ __forceinline__ void f8_offsets(int row0, int lane, uint32_t block_bytes, uint32_t (&ko)[NSUB],
                                           uint32_t (&vo)[NSUB][4]) {
  using C = DecodeF8Cfg<D>;
  const int r = lane >> 2, cq = lane & 3;
  const int k0 = f8_row<D>(2 * cq), k1 = f8_row<D>(2 * cq + 1);
#pragma unroll
  for (int u = 0; u < NSUB; ++u) {
    const int base = row0 + 16 * u;
    ko[u] = swz8<C::ROWB>(base + f8_row<D>((lane & 7) + 8 * ((lane >> 3) & 1)), 16 * (lane >> 4), block_bytes);
    vo[u][0] = swz8<C::ROWB>(base + k0, 4 * r, block_bytes);
    vo[u][1] = swz8<C::ROWB>(base + k1, 4 * r, block_bytes);
    vo[u][2] = swz8<C::ROWB>(base + k0 + 8, 4 * r, block_bytes);
    vo[u][3] = swz8<C::ROWB>(base + k1 + 8, 4 * r, block_bytes);
  }
}

// FP8 counterpart of decode_subtile for NSUB consecutive 16-row sub-tiles
// of a tile stored as swizzled ROWB-byte column blocks (stage bases kst/vst,
// this lane's offsets ko/vo from f8_offsets; with MASK, keys k < n_first and
// k >= n_valid, counted from the first row, are masked, without it all
// 16 NSUB keys are valid), with row scales ksc/vsc from the first row on, Q fragments in f16
// laid out for the byte order ldmatrix delivers (see the kernel), per-head
// score scales hs (scale_log2 * 2^e of heads 2(lane%4), +1), and ev[e] the
// running power of two of head column e's accumulator: O is kept in units of
// 2^ev, ev the largest exponent of any weight p * scale_v seen so far, so
// that the f16 weights p * scale_v * 2^-ev stay below 2 and lose only terms
// under 2^-24 of the largest one. The sub-tiles share one max reduction and
// one exponent reduction, and their independent chains interleave.
template <int D, int NSUB, bool MASK>
__device__ __forceinline__ void decode_subtile_f8(uint32_t kst, uint32_t vst, uint32_t block_bytes,
                                                  const uint32_t (&ko)[NSUB], const uint32_t (&vo)[NSUB][4],
                                                  const float* ksc, const float* vsc, int n_first, int n_valid,
                                                  const uint32_t (&qf)[D / 16][2],
                                                  const float (&hs)[2], float (&m)[2], float (&l)[2],
                                                  float (&o)[D / 16][4], int (&ev)[2], int lane) {
  using C = DecodeF8Cfg<D>;
  const int r = lane >> 2, cq = lane & 3;
  // ---- S^T = K Q^T: ldmatrix over bytes gives lane (r, cq) key rows r, r+8 and
  // code bytes 4cq..4cq+3 (+16) of each 32-byte group; its two 16-bit halves
  // are the two K-steps of the group (the Q fragments follow the same order).
  float c[NSUB][4];
#pragma unroll
  for (int u = 0; u < NSUB; ++u) {
    c[u][0] = c[u][1] = c[u][2] = c[u][3] = 0.f;
#pragma unroll
    for (int grp = 0; grp < D / 32; ++grp) {
      uint32_t r0, r1, r2, r3;
      ldmatrix_x4(grp_addr<C::ROWB>(kst + ko[u], grp, block_bytes), r0, r1, r2, r3);
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        const int sh = 16 * st;
        mma_16816_f16(c[u], f16x2_from_e4m3x2((uint16_t)(r0 >> sh)), f16x2_from_e4m3x2((uint16_t)(r1 >> sh)),
                      f16x2_from_e4m3x2((uint16_t)(r2 >> sh)), f16x2_from_e4m3x2((uint16_t)(r3 >> sh)),
                      qf[2 * grp + st][0], qf[2 * grp + st][1]);
      }
    }
  }
  const int ka = f8_row<D>(r), kb = ka + 8;   // rows (within a sub-tile) of logical keys r, r + 8
  float s[NSUB][4], vsa[NSUB], vsb[NSUB];
#pragma unroll
  for (int u = 0; u < NSUB; ++u) {
    const int a = 16 * u + ka, bq = 16 * u + kb;
    const bool va = !MASK || (a >= n_first && a < n_valid);
    const bool vb = !MASK || (bq >= n_first && bq < n_valid);
    const float ksa = ksc[a], ksb = ksc[bq];
    s[u][0] = va ? c[u][0] * (ksa * hs[0]) : -INFINITY;
    s[u][1] = va ? c[u][1] * (ksa * hs[1]) : -INFINITY;
    s[u][2] = vb ? c[u][2] * (ksb * hs[0]) : -INFINITY;
    s[u][3] = vb ? c[u][3] * (ksb * hs[1]) : -INFINITY;
    // masked rows weigh 0 (their scales may be anything a never-written row holds)
    vsa[u] = va ? vsc[a] : 0.f;
    vsb[u] = vb ? vsc[bq] : 0.f;
  }
  float pw[NSUB][4], alpha[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) mx = fmaxf(mx, fmaxf(s[u][e], s[u][2 + e]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(m[e], mx);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    alpha[e] = ex2(m[e] - m_use);
    float add = 0.f;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) {
      const float pa = ex2(s[u][e] - m_use), pb = ex2(s[u][2 + e] - m_use);
      add += pa + pb;
      pw[u][e] = pa * vsa[u];
      pw[u][2 + e] = pb * vsb[u];
    }
    l[e] = l[e] * alpha[e] + add;
    m[e] = m_new;
  }
  // ---- weights p * scale_v relative to the head's power of two 2^ev (ev
  // never shrinks, so the rescale of O is at most 1)
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float mx = 0.f;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) mx = fmaxf(mx, fmaxf(pw[u][e], pw[u][2 + e]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    int ev_new = ev[e];
    if (mx > 0.f) {
      const int x = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127;   // -127 for subnormals
      ev_new = x > ev_new ? x : ev_new;
    }
    const int dv = ev[e] - ev_new;                                       // <= 0
    const float fo = dv < -126 ? 0.f : __uint_as_float((uint32_t)(127 + dv) << 23);
    const float inv = __uint_as_float((uint32_t)(127 - ev_new) << 23);   // 2^-ev_new
    ev[e] = ev_new;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) {
      pw[u][e] *= inv;
      pw[u][2 + e] *= inv;
    }
    const float ao = alpha[e] * fo;
    // the accumulators move only when a maximum or a power of two changed
    if (__any_sync(0xffffffffu, ao != 1.f)) {
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        o[md][e] *= ao;
        o[md][2 + e] *= ao;
      }
    }
  }
  // ---- O^T += V^T P'^T: lane (r, cq) reads one 32-bit word (code bytes
  // 4r..4r+3 of a 32-byte group) from each of the rows of logical keys 2cq,
  // 2cq+1, 2cq+8, 2cq+9 and regroups the bytes into the A fragments of two
  // 16-row blocks of d: block A holds d = 32 grp + 4r + {0, 1}, block B
  // d = 32 grp + 4r + {2, 3} (rows r and r + 8 of the fragment).
  const int k0 = f8_row<D>(2 * cq), k1 = f8_row<D>(2 * cq + 1), k2 = k0 + 8, k3 = k1 + 8;
#pragma unroll
  for (int u = 0; u < NSUB; ++u) {
    const uint32_t b01 = movmatrix_trans(pack_f16(pw[u][0], pw[u][1]));
    const uint32_t b23 = movmatrix_trans(pack_f16(pw[u][2], pw[u][3]));
    const int t0 = 16 * u + k0, t1 = 16 * u + k1, t2 = 16 * u + k2, t3 = 16 * u + k3;
    const bool u0 = !MASK || (t0 >= n_first && t0 < n_valid), u1 = !MASK || (t1 >= n_first && t1 < n_valid);
    const bool u2 = !MASK || (t2 >= n_first && t2 < n_valid), u3 = !MASK || (t3 >= n_first && t3 < n_valid);
#pragma unroll
    for (int grp = 0; grp < D / 32; ++grp) {
      uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;   // rows never written may hold NaN codes
      if (u0) w0 = ld_shared_u32(grp_addr<C::ROWB>(vst + vo[u][0], grp, block_bytes));
      if (u1) w1 = ld_shared_u32(grp_addr<C::ROWB>(vst + vo[u][1], grp, block_bytes));
      if (u2) w2 = ld_shared_u32(grp_addr<C::ROWB>(vst + vo[u][2], grp, block_bytes));
      if (u3) w3 = ld_shared_u32(grp_addr<C::ROWB>(vst + vo[u][3], grp, block_bytes));
      const uint32_t x01a = __byte_perm(w0, w1, 0x5140), x23a = __byte_perm(w2, w3, 0x5140);
      const uint32_t x01b = __byte_perm(w0, w1, 0x7362), x23b = __byte_perm(w2, w3, 0x7362);
      mma_16816_f16(o[2 * grp], f16x2_from_e4m3x2((uint16_t)x01a), f16x2_from_e4m3x2((uint16_t)(x01a >> 16)),
                    f16x2_from_e4m3x2((uint16_t)x23a), f16x2_from_e4m3x2((uint16_t)(x23a >> 16)), b01, b23);
      mma_16816_f16(o[2 * grp + 1], f16x2_from_e4m3x2((uint16_t)x01b),
                    f16x2_from_e4m3x2((uint16_t)(x01b >> 16)), f16x2_from_e4m3x2((uint16_t)x23b),
                    f16x2_from_e4m3x2((uint16_t)(x23b >> 16)), b01, b23);
    }
  }
}

// The query words (bf16 pairs) one lane of a consumer warp holds as MMA
// B-fragment registers: word j covers dims base(j) + lane_off + {0, 1}, with
// lane_off = 2 (lane % 4) for a bf16 cache and 4 (lane % 4) for FP8. Every
// dim below D/2 and its RoPE partner (+ D/2) sit in the same lane, in words
// j and partner(j).
template <int D, bool F8>
struct QWords {
  static constexpr int NW = D / 8;
  __host__ __device__ static constexpr int base(int j) {
    return F8 ? 32 * (j >> 2) + 16 * (j & 1) + 2 * ((j >> 1) & 1) : 16 * (j >> 1) + 8 * (j & 1);
  }
  __host__ __device__ static constexpr int partner(int j) {
    if (base(j) >= D / 2) return -1;
    for (int k = 0; k < NW; ++k)
      if (base(k) == base(j) + D / 2) return k;
    return -2;
  }
  __host__ __device__ static constexpr bool closed() {
    for (int j = 0; j < NW; ++j)
      if (partner(j) == -2) return false;
    return true;
  }
  static_assert(closed(), "every lower-half query dim has its RoPE partner in the same lane");
};

// Loads one lane's query words and rotates them at the table row given by
// ctab/stab (correctly rounded bf16, rope_pair2). All loads are issued before
// the first is used.
template <int D, bool F8>
__device__ __forceinline__ void load_q_words(const __nv_bfloat16* qrow, int lane_off, const float* ctab,
                                             const float* stab, int rope, uint32_t (&w)[D / 8]) {
  using QW = QWords<D, F8>;
#pragma unroll
  for (int j = 0; j < QW::NW; ++j) w[j] = *reinterpret_cast<const uint32_t*>(qrow + QW::base(j) + lane_off);
  if (rope) {
    float2 cs[QW::NW], sn[QW::NW];
#pragma unroll
    for (int j = 0; j < QW::NW; ++j) {
      if (QW::partner(j) >= 0) {
        cs[j] = *reinterpret_cast<const float2*>(ctab + QW::base(j) + lane_off);
        sn[j] = *reinterpret_cast<const float2*>(stab + QW::base(j) + lane_off);
      }
    }
#pragma unroll
    for (int j = 0; j < QW::NW; ++j) {
      if (QW::partner(j) >= 0) rope_pair2(w[j], w[QW::partner(j)], cs[j].x, cs[j].y, sn[j].x, sn[j].y);
    }
  }
}

// tmK/tmV: the cache's K/V (bf16 elements, or FP8 code bytes); tmKS/tmVS
// (FP8 only): the row scales, dims {rows, n_kv, B, 1}, box {R, 1, 1, 1}.
template <int D, bool F8>
__global__ void __launch_bounds__(288, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKS, const __grid_constant__ CUtensorMap tmVS,
                  const DecodeParams p) {
  using C = DecodeCfgT<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) -> uint32_t { return bar0 + 8u * (uint32_t)s; };
  auto empty_bar = [&](int s) -> uint32_t { return bar0 + 8u * (uint32_t)(C::NS + s); };
  const uint32_t merge_bar = sbase + C::OFF_MBAR;
  volatile int* flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  // flag[0]: abort, flag[1]: "this CTA merges the splits"
  float* sink_sm = reinterpret_cast<float*>(smem + C::OFF_SINK);   // [q_mult] sinks, log2 units
  // position of each ring slot's first row, or -1: the producer has no more stages
  volatile long long* srow = reinterpret_cast<volatile long long*>(smem + C::OFF_SROW);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;      // KV heads of one split run side by side (same cache rows)
  const int split = blockIdx.y;
  const int b = blockIdx.z;
  const int QM = p.q_mult;
  constexpr int HALF = D / 2;

  // Stages (R rows from position lo + sidx R) of this (b, g): the split's
  // static ones first, then dynamic ones while any are left, so CTAs that
  // stream faster take more and all of them finish at about the same time.
  const int F = p.static_stages;
  const long long s_begin = (long long)split * F;
  const bool dyn = (long long)p.S * F < p.n_blocks;
  const bool last_split = split == p.S - 1;

  // The next layer's launch may take this CTA's slot as soon as it frees up;
  // it does its own set-up there and then waits for this grid to complete.
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::NCW);
    }
    mbar_init(merge_bar, 1);
    flag[0] = 0;
    flag[1] = 0;
    fence_barrier_init();
  }
  // The first stages of this split go into L2 while the kernel before this
  // one is still draining (its tail, or a short band layer). A prefetch
  // brings nothing into the SM, so it is safe even if that kernel writes
  // some of these rows: L2 is where its writes land.
  if (warp == C::NCW && lane == 0 && p.n_blocks > 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if constexpr (F8) {
      tma_prefetch_desc(&tmKS);
      tma_prefetch_desc(&tmVS);
    }
    const int pf = F < p.pf_stages ? F : p.pf_stages;
    for (int it = 0; it < pf; ++it) {
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx) {
        const long long pos = p.lo + (s_begin + it) * C::R + 128 * bx;
        const int row = (int)(p.ring_cap > 0 ? pos % p.ring_cap : pos);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_prefetch_l2_4d(&tmK, cb * C::BLKCOLS, row, g, b);
          tma_prefetch_l2_4d(&tmV, cb * C::BLKCOLS, row, g, b);
        }
        if constexpr (F8) {
          tma_prefetch_l2_4d(&tmKS, row, g, b, 0);
          tma_prefetch_l2_4d(&tmVS, row, g, b, 0);
        }
      }
    }
  }
  // The small inputs the consumers read first (the group's query rows, the
  // RoPE table rows at `off`, the sinks, the new K/V row) go into L2 too:
  // lane i of warp 0 takes the i-th 128-byte line of that list.
  if (warp == 0) {
    constexpr int LPR = (D * 2 + 127) / 128;   // lines per bf16 row
    const int QM_ = p.q_mult;
    const char* a = nullptr;
    int i = lane;
    if (i < QM_ * LPR) {
      a = reinterpret_cast<const char*>(p.q + b * p.qs0 + (long long)(g * QM_ + i / LPR) * p.qs2) + 128 * (i % LPR);
    } else if ((i -= QM_ * LPR) < 2 * LPR) {
      if (p.rope) a = reinterpret_cast<const char*>((i < LPR ? p.cos_t : p.sin_t) + p.off * (D / 2)) + 128 * (i % LPR);
    } else if ((i -= 2 * LPR) < 2 * LPR) {
      if (split == p.S - 1)
        a = reinterpret_cast<const char*>(i < LPR ? p.k + b * p.ks0 + (long long)g * p.ks2
                                                  : p.v + b * p.vs0 + (long long)g * p.vs2) + 128 * (i % LPR);
    } else if (i == 2 * LPR) {
      if (p.sinks) a = reinterpret_cast<const char*>(p.sinks + g * QM_);
    }
    if (a) prefetch_l2(a);
  }
  __syncthreads();
  // Everything below reads or writes global memory (q, the cache, the split
  // workspace, the output), which the kernel before this one may still be using.
  griddep_wait();

  if (warp == C::NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int* grab = p.ws_grab + (b * p.n_kv + g);
      int pending = dyn ? atomicAdd(grab, 1) : 0;   // the first dynamic stage, asked for early
      int it = 0;
      for (int k = 0; !flag[0]; ++k) {
        long long sidx;
        if (k < F) {
          sidx = s_begin + k;
        } else {
          if (!dyn) break;
          sidx = (long long)p.S * F + pending;
          if (sidx >= p.n_blocks) break;
          pending = atomicAdd(grab, 1);   // the next one, in flight while this stage loads
        }
        const int s = it % C::NS;
        if (!mbar_wait(empty_bar(s), (uint32_t)(((it / C::NS) & 1) ^ 1))) { flag[0] = 1; break; }
        const long long pos0 = p.lo + sidx * C::R;
        srow[s] = pos0;
        mbar_arrive_expect_tx(full_bar(s), C::STAGE_TX);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) {
          // boxes of 128 rows: none wraps a ring (ring stages start on multiples of 128)
          const long long pos = pos0 + 128 * bx;
          const int row = (int)(p.ring_cap > 0 ? pos % p.ring_cap : pos);
          const uint32_t boff = (uint32_t)bx * 128u * (C::BLOCK_BYTES / C::R);
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb) {
            tma_load_4d(sbase + C::OFF_K + s * C::STAGE_BYTES + cb * C::BLOCK_BYTES + boff, &tmK, full_bar(s),
                        cb * C::BLKCOLS, row, g, b);
            tma_load_4d(sbase + C::OFF_V + s * C::STAGE_BYTES + cb * C::BLOCK_BYTES + boff, &tmV, full_bar(s),
                        cb * C::BLKCOLS, row, g, b);
          }
          if constexpr (F8) {
            // row is a multiple of 128 (the FP8 launch aligns every stage), so
            // the innermost coordinate of these fp32 boxes is 16-byte aligned
            tma_load_4d(sbase + C::OFF_KS + s * C::R * 4 + bx * 512, &tmKS, full_bar(s), row, g, b, 0);
            tma_load_4d(sbase + C::OFF_VS + s * C::R * 4 + bx * 512, &tmVS, full_bar(s), row, g, b, 0);
          }
        }
        ++it;
      }
      // the end of this CTA's stream: a slot marked -1, completed by a plain arrive
      if (!flag[0]) {
        const int s = it % C::NS;
        if (mbar_wait(empty_bar(s), (uint32_t)(((it / C::NS) & 1) ^ 1))) {
          srow[s] = -1;
          mbar_arrive(full_bar(s));
        } else {
          flag[0] = 1;
        }
      }
      if (flag[0]) {
        for (int j = (it > C::NS ? it - C::NS : 0); j < it; ++j)
          mbar_wait_drain(full_bar(j % C::NS), (uint32_t)((j / C::NS) & 1));
      }
    }
    return;  // the producer takes no part in the merge (named barriers below count 32*NCW)
  }

  // ---------------------------------------------------------------- consumers
  // Every global load a consumer warp needs before its first tile goes out
  // at once, so their latencies overlap: the sinks (into smem), the query
  // words and, in warp 0 of the last split, the new K/V row with its RoPE
  // table entries.
  // (the sink goes to smem only after the query words have arrived, so its
  // load does not hold up theirs)
  const float sink_in = (threadIdx.x < QM && p.sinks) ? p.sinks[g * QM + threadIdx.x] : -INFINITY;
  const bool new_row = last_split && warp == 0;
  const long long new_slot = p.ring_cap > 0 ? p.off % p.ring_cap : p.off;
  const long long new_crow = ((long long)b * p.n_kv + g) * p.cap + new_slot;
  const __nv_bfloat16* krow = p.k + b * p.ks0 + (long long)g * p.ks2;
  const __nv_bfloat16* vrow = p.v + b * p.vs0 + (long long)g * p.vs2;
  const float* ctab = p.cos_t + p.off * HALF;
  const float* stab = p.sin_t + p.off * HALF;
  // bf16 cache: unit u < HALF/2 of a lane is K word pair (2u, 2u + HALF),
  // unit u >= HALF/2 the same pair of V. FP8 cache: the lane's words 2 lane
  // + 64 i (the quantiser's layout) and, for K, their RoPE partners.
  constexpr int NRU = F8 ? 2 : (HALF + 31) / 32;
  uint32_t nr_a[NRU], nr_b[NRU], nr_v[NRU];
  float2 nr_c[NRU], nr_s[NRU];
  if (new_row) {
#pragma unroll
    for (int i = 0; i < NRU; ++i) {
      nr_a[i] = nr_b[i] = nr_v[i] = 0u;
      nr_c[i] = nr_s[i] = make_float2(0.f, 0.f);
      if constexpr (F8) {
        const int c = 2 * lane + 64 * i;
        if (c < D) {
          const int i0 = c < HALF ? c : c - HALF;
          nr_a[i] = *reinterpret_cast<const uint32_t*>(krow + i0);
          nr_b[i] = *reinterpret_cast<const uint32_t*>(krow + i0 + HALF);
          nr_v[i] = *reinterpret_cast<const uint32_t*>(vrow + c);
          if (p.rope) {
            nr_c[i] = *reinterpret_cast<const float2*>(ctab + i0);
            nr_s[i] = *reinterpret_cast<const float2*>(stab + i0);
          }
        }
      } else {
        const int u = lane + 32 * i;
        if (u < HALF) {
          const bool is_v = u >= HALF / 2;
          const int c = 2 * (is_v ? u - HALF / 2 : u);
          const __nv_bfloat16* row = is_v ? vrow : krow;
          nr_a[i] = *reinterpret_cast<const uint32_t*>(row + c);
          nr_b[i] = *reinterpret_cast<const uint32_t*>(row + c + HALF);
          if (!is_v && p.rope) {
            nr_c[i] = *reinterpret_cast<const float2*>(ctab + c);
            nr_s[i] = *reinterpret_cast<const float2*>(stab + c);
          }
        }
      }
    }
  }

  // Q fragments (B operand, col-major [d][head]): head n = lane/4 of the
  // group, rotated at position off; the lane's words are listed by QWords.
  uint32_t qf[D / 16][2];
  float hs[2] = {0.f, 0.f};   // FP8: score scale of heads 2(lane%4), 2(lane%4)+1
  {
    const int n = lane >> 2;
    const bool hv = n < QM;
    const __nv_bfloat16* qrow = p.q + b * p.qs0 + (long long)(g * QM + (hv ? n : 0)) * p.qs2;
    uint32_t w[D / 8];
    load_q_words<D, F8>(qrow, F8 ? 4 * (lane & 3) : 2 * (lane & 3), ctab, stab, p.rope, w);
    if constexpr (F8) {
      // FP8 layout: fragment (grp, st) holds dims 32 grp + 4(lane%4) + 2 st + {0,1}
      // (register 0) and the same + 16 (register 1), matching the code bytes
      // ldmatrix hands each lane. Head n is scaled by 2^-e_n so that its
      // largest |q| lies in [2^14, 2^15): every bf16 q is then exact in f16
      // down to 2^-29 of that maximum.
      float qv[D / 16][2][2];
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        qv[j >> 1][j & 1][0] = hv ? bf16_lo(w[j]) : 0.f;
        qv[j >> 1][j & 1][1] = hv ? bf16_hi(w[j]) : 0.f;
        amax = fmaxf(amax, fmaxf(fabsf(qv[j >> 1][j & 1][0]), fabsf(qv[j >> 1][j & 1][1])));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      int eq = 0;
      if (amax > 0.f) {
        eq = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 14;
        eq = eq < -110 ? -110 : (eq > 110 ? 110 : eq);
      }
      const float down = __uint_as_float((uint32_t)(127 - eq) << 23);
#pragma unroll
      for (int f = 0; f < D / 16; ++f)
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) qf[f][hlf] = pack_f16(qv[f][hlf][0] * down, qv[f][hlf][1] * down);
      const float hs_mine = p.scale_log2 * __uint_as_float((uint32_t)(127 + eq) << 23);
      hs[0] = __shfl_sync(0xffffffffu, hs_mine, 8 * (lane & 3));
      hs[1] = __shfl_sync(0xffffffffu, hs_mine, 8 * (lane & 3) + 4);
    } else {
#pragma unroll
      for (int j = 0; j < D / 8; ++j) qf[j >> 1][j & 1] = hv ? w[j] : 0u;
    }
  }
  if (threadIdx.x < QM) sink_sm[threadIdx.x] = sink_in * 1.4426950408889634f;
  int ev[2] = {-127, -127};   // FP8: powers of two of the two head columns' accumulators
  // FP8: this lane's shared-memory offsets within a stage (the same for every stage)
  uint32_t f8ko[C::RW / 16], f8vo[C::RW / 16][4];
  if constexpr (F8) f8_offsets<D, C::RW / 16>(C::RW * warp, lane, C::BLOCK_BYTES, f8ko, f8vo);

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[D / 16][4];
#pragma unroll
  for (int md = 0; md < D / 16; ++md) o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;

  // The new row: rotate k, write K/V row `off` of the cache, stage it in smem
  // as row 0 of a zeroed 16-row tile. An FP8 cache stores (and this call
  // attends) the row quantised.
  if (new_row) {
    uint8_t* xk = smem + C::OFF_XK;
    uint8_t* xv = smem + C::OFF_XV;
    for (int idx = lane; idx < (int)(C::XTILE / 16); idx += 32) {
      reinterpret_cast<uint4*>(xk)[idx] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(xv)[idx] = make_uint4(0, 0, 0, 0);
    }
    if constexpr (F8) {
      float* xs = reinterpret_cast<float*>(smem + C::OFF_XS);
      xs[lane] = 0.f;
      __syncwarp();
      float xkv[2][2], xvv[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int c = 2 * lane + 64 * i;
        uint32_t kw = c < HALF ? nr_a[i] : nr_b[i];
        if (c < D && p.rope) {
          uint32_t w1 = nr_a[i], w2 = nr_b[i];
          rope_pair2(w1, w2, nr_c[i].x, nr_c[i].y, nr_s[i].x, nr_s[i].y);
          kw = c < HALF ? w1 : w2;
        }
        xkv[i][0] = bf16_lo(kw);
        xkv[i][1] = bf16_hi(kw);
        xvv[i][0] = bf16_lo(nr_v[i]);
        xvv[i][1] = bf16_hi(nr_v[i]);
      }
      uint16_t kc[2], vc[2];
      const float sk = quantize_row_warp<2>(xkv, D, reinterpret_cast<uint8_t*>(p.ck) + new_crow * D, lane, kc);
      const float sv = quantize_row_warp<2>(xvv, D, reinterpret_cast<uint8_t*>(p.cv) + new_crow * D, lane, vc);
      if (lane == 0) {
        p.cks[new_crow] = sk;
        p.cvs[new_crow] = sv;
        xs[0] = sk;
        xs[16] = sv;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int c = 2 * lane + 64 * i;
        if (c < D) {
          *reinterpret_cast<uint16_t*>(xk + swz8<C::ROWB>(0, c, C::XBLOCK)) = kc[i];
          *reinterpret_cast<uint16_t*>(xv + swz8<C::ROWB>(0, c, C::XBLOCK)) = vc[i];
        }
      }
    } else {
      __syncwarp();
      __nv_bfloat16* ckrow = p.ck + new_crow * D;
      __nv_bfloat16* cvrow = p.cv + new_crow * D;
#pragma unroll
      for (int i = 0; i < NRU; ++i) {
        const int u = lane + 32 * i;
        if (u < HALF) {
          const bool is_v = u >= HALF / 2;
          const int c = 2 * (is_v ? u - HALF / 2 : u);
          uint32_t w1 = nr_a[i], w2 = nr_b[i];
          if (!is_v && p.rope) rope_pair2(w1, w2, nr_c[i].x, nr_c[i].y, nr_s[i].x, nr_s[i].y);
          __nv_bfloat16* crow = is_v ? cvrow : ckrow;
          uint8_t* tile = is_v ? xv : xk;
          *reinterpret_cast<uint32_t*>(crow + c) = w1;
          *reinterpret_cast<uint32_t*>(crow + c + HALF) = w2;
          *reinterpret_cast<uint32_t*>(tile + swz_off<C::CB>(0, c, C::XBLOCK)) = w1;
          *reinterpret_cast<uint32_t*>(tile + swz_off<C::CB>(0, c + HALF, C::XBLOCK)) = w2;
        }
      }
    }
    __syncwarp();
  }

  for (int it = 0;; ++it) {
    const int s = it % C::NS;
    if (!mbar_wait(full_bar(s), (uint32_t)((it / C::NS) & 1))) { flag[0] = 1; break; }
    const long long pos0 = srow[s];
    if (pos0 < 0) break;   // the producer's end mark
    const long long row0 = pos0 + C::RW * warp;
    const long long nv = p.off - row0;
    const long long nf = p.lo_mask - row0;
    if (nv > 0 && nf < C::RW && !flag[0]) {
      if constexpr (F8) {
        const uint32_t kst = sbase + C::OFF_K + s * C::STAGE_BYTES, vst = sbase + C::OFF_V + s * C::STAGE_BYTES;
        const float* ks = reinterpret_cast<const float*>(smem + C::OFF_KS) + s * C::R + C::RW * warp;
        const float* vs = reinterpret_cast<const float*>(smem + C::OFF_VS) + s * C::R + C::RW * warp;
        if (nf <= 0 && nv >= C::RW)
          decode_subtile_f8<D, C::RW / 16, false>(kst, vst, C::BLOCK_BYTES, f8ko, f8vo, ks, vs, 0, C::RW, qf, hs,
                                                  m, l, o, ev, lane);
        else
          decode_subtile_f8<D, C::RW / 16, true>(kst, vst, C::BLOCK_BYTES, f8ko, f8vo, ks, vs,
                                                 nf > 0 ? (int)nf : 0, nv > C::RW ? C::RW : (int)nv, qf, hs, m,
                                                 l, o, ev, lane);
      } else
        decode_subtile<D>(sbase + C::OFF_K + s * C::STAGE_BYTES, sbase + C::OFF_V + s * C::STAGE_BYTES,
                          C::BLOCK_BYTES, 16 * warp, nf > 0 ? (int)nf : 0, nv > 16 ? 16 : (int)nv, qf,
                          p.scale_log2, m, l, o, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }
  if (last_split && warp == 0) {
    if constexpr (F8) {
      const float* xs = reinterpret_cast<const float*>(smem + C::OFF_XS);
      uint32_t xko[1], xvo[1][4];
      f8_offsets<D, 1>(0, lane, C::XBLOCK, xko, xvo);
      decode_subtile_f8<D, 1, true>(sbase + C::OFF_XK, sbase + C::OFF_XV, C::XBLOCK, xko, xvo, xs, xs + 16, 0, 1,
                                    qf, hs, m, l, o, ev, lane);
    } else {
      decode_subtile<D>(sbase + C::OFF_XK, sbase + C::OFF_XV, C::XBLOCK, 0, 0, 1, qf, p.scale_log2, m, l,
                        o, lane);
    }
  }

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
    if constexpr (F8) {
      // fragment rows r, r + 8 of block md are d = 32(md/2) + 4r + 2(md%2) + {0, 1};
      // head column e's accumulators are in units of 2^ev[e]
      const float f0 = ldexpf(1.0f, ev[0]), f1 = ldexpf(1.0f, ev[1]);
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        const int d0 = 32 * (md >> 1) + 4 * (lane >> 2) + 2 * (md & 1);
        rw[16 + (2 * t) * D + d0] = o[md][0] * f0;
        rw[16 + (2 * t + 1) * D + d0] = o[md][1] * f1;
        rw[16 + (2 * t) * D + d0 + 1] = o[md][2] * f0;
        rw[16 + (2 * t + 1) * D + d0 + 1] = o[md][3] * f1;
      }
    } else {
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        const int d0 = md * 16 + (lane >> 2);
        rw[16 + (2 * t) * D + d0] = o[md][0];
        rw[16 + (2 * t + 1) * D + d0] = o[md][1];
        rw[16 + (2 * t) * D + d0 + 8] = o[md][2];
        rw[16 + (2 * t + 1) * D + d0 + 8] = o[md][3];
      }
    }
  }
  named_bar_sync(1, 32 * C::NCW);

  const float LN2 = 0.6931471805599453f;
  const int tid = threadIdx.x;  // 0 .. 32*NCW-1
  constexpr int NT = 32 * C::NCW;
  const int RF = p.rec_floats;
  float* rec = p.ws_rec + (((long long)b * p.n_kv + g) * p.S + split) * RF;
  // two adjacent outputs (head n, dims d, d+1) per thread and pass
  for (int idx = 2 * tid; idx < QM * D; idx += 2 * NT) {
    const int n = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::NCW; ++w) M = fmaxf(M, red[w * (C::RED_WARP / 4) + n]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O0 = 0.f, O1 = 0.f;
#pragma unroll
    for (int w = 0; w < C::NCW; ++w) {
      const float* rw = red + w * (C::RED_WARP / 4);
      const float f = ex2(rw[n] - Mu);
      L += rw[8 + n] * f;
      const float2 ov = *reinterpret_cast<const float2*>(rw + 16 + n * D + d);
      O0 += ov.x * f;
      O1 += ov.y * f;
    }
    const int h = g * QM + n;
    if (p.S == 1) {
      const float sink2 = sink_sm[n];
      const float M2 = fmaxf(M, sink2);
      const float fo = ex2(M - M2);
      const float tot = L * fo + ex2(sink2 - M2);
      *reinterpret_cast<uint32_t*>(p.out + b * p.os0 + (long long)h * p.os2 + d) =
          pack_bf16(O0 * fo / tot, O1 * fo / tot);
      if (d == 0 && p.lse) p.lse[(long long)b * p.n_q + h] = (M2 + __log2f(tot)) * LN2;
    } else {
      *reinterpret_cast<float2*>(rec + n * D + d) = make_float2(O0, O1);
      if (d == 0) {
        rec[QM * D + n] = M;
        rec[QM * D + QM + n] = L;
      }
    }
  }
  if (p.S == 1) return;

  // The ticket: the barrier orders every thread's record stores before
  // thread 0's release; its acquire makes the other CTAs' records visible to
  // the merging CTA (whose thread 0 alone reads them, by bulk copy).
  named_bar_sync(1, NT);
  if (tid == 0) {
    const int ticket = atom_add_acq_rel_gpu(p.ws_cnt + (b * p.n_kv + g), 1);
    flag[1] = (ticket == p.S - 1) ? 1 : 0;
  }
  named_bar_sync(1, NT);
  if (!flag[1]) return;

  // Merge the S records of (b, g). The K/V ring is idle now: one bulk copy
  // per round brings as many records as it holds (normally all S) into it,
  // so the tail pays one memory round trip instead of one per batch of
  // loads. A group of G adjacent lanes owns four outputs (head n, dims
  // d .. d+3); its lanes take every G-th record and combine by shuffles.
  // The running maximum starts at the sink (log2 units):
  // M = max(sink, m_s), l = e^{sink-M} + sum_s e^{m_s-M} l_s.
  const int S = p.S;
  const uint32_t rec_bytes = (uint32_t)RF * 4u;
  const int per_round = (int)(C::RING_BYTES / rec_bytes);
  const float* recs = reinterpret_cast<const float*>(smem);
  const char* gsrc = reinterpret_cast<const char*>(p.ws_rec + ((long long)b * p.n_kv + g) * S * RF);
  const int nf4 = QM * D / 4;
  const int G = 2 * nf4 <= NT ? 2 : 1;   // lanes per output group
  const int f4 = tid / G, part = tid % G;
  const bool owner = f4 < nf4;
  const int n = owner ? (4 * f4) / D : 0;
  const int d = owner ? (4 * f4) % D : 0;
  const int om = QM * D + n, ol = QM * D + QM + n, oo = n * D + d;
  float M = sink_sm[n];
  float L = (M == -INFINITY) ? 0.f : 1.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0, r = 0; s0 < S; s0 += per_round, ++r) {
    const int cnt = S - s0 < per_round ? S - s0 : per_round;
    if (tid == 0) {
      // the records were written by generic stores (other CTAs', acquired
      // through the ticket) and the ring was last written the same way
      fence_proxy_async_global();
      fence_proxy_async_smem();
      const uint32_t bytes = (uint32_t)cnt * rec_bytes;
      mbar_arrive_expect_tx(merge_bar, bytes);
      for (uint32_t o = 0; o < bytes; o += 32768u)
        bulk_load(sbase + o, gsrc + (size_t)s0 * rec_bytes + o, bytes - o < 32768u ? bytes - o : 32768u,
                  merge_bar);
    }
    // a wait that runs out is recorded in the status word; the copy is then
    // drained before the ring is read or this CTA exits
    if (!mbar_wait(merge_bar, (uint32_t)(r & 1))) mbar_wait_drain(merge_bar, (uint32_t)(r & 1));
    float Mr = M;
    float4 ar = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lr = 0.f;
    if (owner) {
      float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
      int s2 = part;
      for (; s2 + 3 * G < cnt; s2 += 4 * G) {
        m0 = fmaxf(m0, recs[s2 * RF + om]);
        m1 = fmaxf(m1, recs[(s2 + G) * RF + om]);
        m2 = fmaxf(m2, recs[(s2 + 2 * G) * RF + om]);
        m3 = fmaxf(m3, recs[(s2 + 3 * G) * RF + om]);
      }
      for (; s2 < cnt; s2 += G) m0 = fmaxf(m0, recs[s2 * RF + om]);
      Mr = fmaxf(fmaxf(Mr, fmaxf(m0, m1)), fmaxf(m2, m3));
    }
    if (G == 2) Mr = fmaxf(Mr, __shfl_xor_sync(0xffffffffu, Mr, 1));
    const float Mu = (Mr == -INFINITY) ? 0.f : Mr;
    if (owner) {
#pragma unroll 4
      for (int s2 = part; s2 < cnt; s2 += G) {
        const float* rr = recs + s2 * RF;
        const float w = ex2(rr[om] - Mu);
        Lr = fmaf(w, rr[ol], Lr);
        const float4 v = *reinterpret_cast<const float4*>(rr + oo);
        ar.x = fmaf(w, v.x, ar.x);
        ar.y = fmaf(w, v.y, ar.y);
        ar.z = fmaf(w, v.z, ar.z);
        ar.w = fmaf(w, v.w, ar.w);
      }
    }
    if (G == 2) {
      Lr += __shfl_xor_sync(0xffffffffu, Lr, 1);
      ar.x += __shfl_xor_sync(0xffffffffu, ar.x, 1);
      ar.y += __shfl_xor_sync(0xffffffffu, ar.y, 1);
      ar.z += __shfl_xor_sync(0xffffffffu, ar.z, 1);
      ar.w += __shfl_xor_sync(0xffffffffu, ar.w, 1);
    }
    const float f = ex2(M - Mu);
    L = fmaf(L, f, Lr);
    acc.x = fmaf(acc.x, f, ar.x);
    acc.y = fmaf(acc.y, f, ar.y);
    acc.z = fmaf(acc.z, f, ar.z);
    acc.w = fmaf(acc.w, f, ar.w);
    M = Mr;
    named_bar_sync(1, NT);   // the ring is read before the next round's copy overwrites it
  }
  if (owner && part == 0) {
    const int h = g * QM + n;
    const float inv = 1.0f / L;
    uint2 packed;
    packed.x = pack_bf16(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(p.out + b * p.os0 + (long long)h * p.os2 + d) = packed;
    if (d == 0 && p.lse) p.lse[(long long)b * p.n_q + h] = (M + __log2f(L)) * LN2;
  }
  if (tid == 0) {
    p.ws_cnt[b * p.n_kv + g] = 0;
    p.ws_grab[b * p.n_kv + g] = 0;
  }
}

}  // namespace sa
