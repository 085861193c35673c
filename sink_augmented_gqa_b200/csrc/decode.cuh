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
  long long chunk;  // cache rows per split (multiple of 128)
  float* cks;       // FP8 caches: row scales [B][n_kv][cap] of K and of V
  float* cvs;
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
  static constexpr uint32_t OFF_BAR = OFF_XS + 128;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 8 * (2 * NS) + 16 + 1024;
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
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
      o[md][e] *= ao;
      o[md][2 + e] *= ao;
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

  // The next layer's launch may take this CTA's slot as soon as it frees up;
  // it does its own set-up there and then waits for this grid to complete.
  griddep_launch_dependents();
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
  // Everything below reads or writes global memory (q, the cache, the split
  // workspace, the output), which the kernel before this one may still be using.
  griddep_wait();

  if (warp == C::NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_stages > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if constexpr (F8) {
        tma_prefetch_desc(&tmKS);
        tma_prefetch_desc(&tmVS);
      }
      int issued = 0;
      for (int it = 0; it < n_stages; ++it) {
        const int s = it % C::NS;
        if (!mbar_wait(empty_bar(s), (uint32_t)(((it / C::NS) & 1) ^ 1))) { flag[0] = 1; break; }
        mbar_arrive_expect_tx(full_bar(s), C::STAGE_TX);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) {
          // boxes of 128 rows: none wraps a ring (ring stages start on multiples of 128)
          const long long pos = r_begin + (long long)it * C::R + 128 * bx;
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
  float hs[2] = {0.f, 0.f};   // FP8: score scale of heads 2(lane%4), 2(lane%4)+1
  if constexpr (F8) {
    // FP8 layout: fragment (grp, st) holds dims 32 grp + 4(lane%4) + 2 st + {0,1}
    // (register 0) and the same + 16 (register 1), matching the code bytes
    // ldmatrix hands each lane. Head n is scaled by 2^-e_n so that its
    // largest |q| lies in [2^14, 2^15): every bf16 q is then exact in f16
    // down to 2^-29 of that maximum.
    const int n = lane >> 2;
    const bool hv = n < QM;
    const __nv_bfloat16* qrow = p.q + b * p.qs0 + (long long)(g * QM + (hv ? n : 0)) * p.qs2;
    const float* cs = p.cos_t + p.off * HALF;
    const float* sn = p.sin_t + p.off * HALF;
    float qv[D / 16][2][2];
    float amax = 0.f;
#pragma unroll
    for (int f = 0; f < D / 16; ++f) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 32 * (f >> 1) + 16 * hlf + 4 * (lane & 3) + 2 * (f & 1) + e;
          float x = __bfloat162float(qrow[c]);
          if (p.rope) {
            const int i = c < HALF ? c : c - HALF;
            uint32_t y1, y2;
            rope_pair(__bfloat162float(qrow[i]), __bfloat162float(qrow[i + HALF]), cs[i], sn[i], y1, y2);
            x = __uint_as_float((c < HALF ? y1 : y2) << 16);
          }
          x = hv ? x : 0.f;
          qv[f][hlf][e] = x;
          amax = fmaxf(amax, fabsf(x));
        }
      }
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
  int ev[2] = {-127, -127};   // FP8: powers of two of the two head columns' accumulators
  // FP8: this lane's shared-memory offsets within a stage (the same for every stage)
  uint32_t f8ko[C::RW / 16], f8vo[C::RW / 16][4];
  if constexpr (F8) f8_offsets<D, C::RW / 16>(C::RW * warp, lane, C::BLOCK_BYTES, f8ko, f8vo);

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[D / 16][4];
#pragma unroll
  for (int md = 0; md < D / 16; ++md) o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;

  // The new row: rotate k, write K/V row `off` of the cache, stage it in smem.
  // An FP8 cache stores (and this call attends) the row quantised.
  if constexpr (F8) {
    if (last_split && warp == 0) {
      uint8_t* xk = smem + C::OFF_XK;
      uint8_t* xv = smem + C::OFF_XV;
      float* xs = reinterpret_cast<float*>(smem + C::OFF_XS);
      const __nv_bfloat16* krow = p.k + b * p.ks0 + (long long)g * p.ks2;
      const __nv_bfloat16* vrow = p.v + b * p.vs0 + (long long)g * p.vs2;
      const long long slot = p.ring_cap > 0 ? p.off % p.ring_cap : p.off;
      const long long crow = ((long long)b * p.n_kv + g) * p.cap + slot;
      for (int idx = lane; idx < (int)(C::XTILE / 16); idx += 32) {
        reinterpret_cast<uint4*>(xk)[idx] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(xv)[idx] = make_uint4(0, 0, 0, 0);
      }
      xs[lane] = 0.f;
      __syncwarp();
      float xkv[2][2], xvv[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 2 * lane + 64 * i + e;
          float kx = 0.f, vx = 0.f;
          if (c < D) {
            kx = __bfloat162float(krow[c]);
            if (p.rope) {
              const int i0 = c < HALF ? c : c - HALF;
              uint32_t y1, y2;
              rope_pair(__bfloat162float(krow[i0]), __bfloat162float(krow[i0 + HALF]),
                        p.cos_t[p.off * HALF + i0], p.sin_t[p.off * HALF + i0], y1, y2);
              kx = __uint_as_float((c < HALF ? y1 : y2) << 16);
            }
            vx = __bfloat162float(vrow[c]);
          }
          xkv[i][e] = kx;
          xvv[i][e] = vx;
        }
      }
      uint16_t kc[2], vc[2];
      const float sk = quantize_row_warp<2>(xkv, D, reinterpret_cast<uint8_t*>(p.ck) + crow * D, lane, kc);
      const float sv = quantize_row_warp<2>(xvv, D, reinterpret_cast<uint8_t*>(p.cv) + crow * D, lane, vc);
      if (lane == 0) {
        p.cks[crow] = sk;
        p.cvs[crow] = sv;
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
      __syncwarp();
    }
  } else if (last_split && warp == 0) {
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
    const long long row0 = r_begin + (long long)it * C::R + C::RW * warp;
    const long long nv = r_end - row0;
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
