// libsinkattn: C ABI, argument validation, cache bookkeeping, tensor-map
// construction and kernel launches. Every declaration lives in
// include/sinkattn.h; this file is the single translation unit of the
// library, so the device status word in ptx.cuh exists once per device.

#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/sinkattn.h"
#include "backward.cuh"
#include "band.cuh"
#include "backward_tc.cuh"
#include "decode.cuh"
#include "fp8.cuh"
#include "gemm.cuh"
#include "prefill.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace {

using sa::DecodeCfg;
using sa::DecodeParams;
using sa::PrefillCfg;
using sa::PrefillParams;

// ---------------------------------------------------------------------------
// Small host helpers
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool strides_ok(const int64_t s[3]) {
  return s != nullptr && s[0] >= 0 && s[1] >= 0 && s[2] >= 0 && s[0] % 8 == 0 && s[1] % 8 == 0 &&
         s[2] % 8 == 0;
}

bool head_dim_ok(int d) { return d == 64 || d == 96 || d == 128; }
// Backward workspace rows per (sequence, head): T rounded up to a multiple of
// 384, so that every streamed query tile (64, 96 or 128 rows) lies inside.
int bwd_rows_padded(int T) { return (T + 383) / 384 * 384; }

// Ring capacity granule: a multiple of every key-tile height the kernels use
// (128 decode rows; 128, 96, 64 prefill keys), so no tile wraps around.
constexpr int kRingQuantum = 384;

// SM count of the current device, looked up once per device (it is read on
// every launch).
int num_sms() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 256 ? 256 : (n < 1 ? 1 : n);
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

int grid_for(long long n) {
  long long blocks = (n + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map over one cache buffer [B][n_kv][cap][d] bf16 that exposes only
// rows [0, rows_valid) (later rows read back as zeros): dims {d, rows, n_kv,
// B}, box {CB, box_rows, 1, 1}.
bool make_cache_map(CUtensorMap* map, void* base, int d, int n_kv, long long rows_valid, int cap,
                    int B, int box_rows, int cb) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows_valid < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows_valid, (cuuint64_t)n_kv, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)cap * d * 2,
                                 (cuuint64_t)n_kv * cap * d * 2};
  const cuuint32_t box[4] = {(cuuint32_t)cb, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         cb == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 caches: tensor map over the codes [B][n_kv][cap][d] bytes exposing rows
// [0, rows_valid), box {rowb, box_rows, 1, 1} swizzled over rowb bytes.
bool make_codes_map(CUtensorMap* map, void* base, int d, int n_kv, long long rows_valid, int cap,
                    int B, int box_rows, int rowb) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows_valid < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows_valid, (cuuint64_t)n_kv, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)cap * d, (cuuint64_t)n_kv * cap * d};
  const cuuint32_t box[4] = {(cuuint32_t)rowb, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle sw = rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : (rowb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 caches: tensor map over the row scales [B][n_kv][cap] fp32 exposing
// rows [0, rows_valid): dims {rows_valid, n_kv, B, 1}, box {box_rows, 1, 1, 1}.
bool make_scales_map(CUtensorMap* map, void* base, int n_kv, long long rows_valid, int cap, int B,
                     int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows_valid < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)rows_valid, (cuuint64_t)n_kv, (cuuint64_t)B, 1};
  const cuuint64_t strides[3] = {(cuuint64_t)cap * 4, (cuuint64_t)n_kv * cap * 4,
                                 (cuuint64_t)B * n_kv * cap * 4};
  const cuuint32_t box[4] = {(cuuint32_t)box_rows, 1, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a row-major bf16 matrix [rows][ld] exposing columns
// [0, cols): dims {cols, rows, 1, 1}, box {box_cols, box_rows, 1, 1}.
bool make_matrix_map(CUtensorMap* map, const void* base, long long cols, long long rows, long long ld,
                     int box_cols, int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows < 1 || cols < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, 1, 1};
  const cuuint64_t strides[3] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * rows, (cuuint64_t)ld * 2 * rows};
  const cuuint32_t box[4] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a strided [B][T][H][d] bf16 activation (inner dim
// contiguous, other strides in elements, multiples of 8): dims {d, T, H, B},
// box {CB, 128, 1, 1} -- one 128-row query tile of one head per CB-wide
// column block; rows past T read as zeros.
bool make_rows_map(CUtensorMap* map, const void* base, int d, int T, int H, int B,
                   const int64_t st[3], int cb, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || T < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)st[1] * 2, (cuuint64_t)st[2] * 2, (cuuint64_t)st[0] * 2};
  const cuuint32_t box[4] = {(cuuint32_t)cb, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         cb == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a dense fp32 [B][T][H][d] array (the backward's dq) whose box
// is box_rows consecutive rows of one head ({d, 1, box_rows, 1} over dims
// {d, H, T, B}): the TMA reduce-add target; rows past T are dropped.
bool make_f32_rows_map(CUtensorMap* map, float* base, int d, int T, int H, int B, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || T < 1) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)T * H * d * 4};
  const cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a strided [B][T][H][d] bf16 activation whose box is
// box_heads consecutive heads of box_rows consecutive rows (d = 64: one
// 128-byte swizzled row per (row, head)): dims {d, H, T, B}, box
// {d, box_heads, box_rows, 1}; rows past T read as zeros and are dropped on
// store.
bool make_heads_map(CUtensorMap* map, const void* base, int d, int T, int H, int B, const int64_t st[3],
                    int box_heads, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || T < 1 || d != 64) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
  const cuuint32_t box[4] = {(cuuint32_t)d, (cuuint32_t)box_heads, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

sa_status last_launch_status() {
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// Cache bookkeeping after an append of T rows at `start`.
void note_append(sa_kv_cache* c, int64_t start, int T) {
  c->seq += 1;
  if (start < c->high_water) {
    if (c->log_len == SA_KV_LOG_CAP) {
      if (c->log_seq[0] > c->log_floor_seq) c->log_floor_seq = c->log_seq[0];
      if (c->log_row[0] < c->log_floor_row) c->log_floor_row = c->log_row[0];
      memmove(c->log_seq, c->log_seq + 1, sizeof(int64_t) * (SA_KV_LOG_CAP - 1));
      memmove(c->log_row, c->log_row + 1, sizeof(int64_t) * (SA_KV_LOG_CAP - 1));
      c->log_len -= 1;
    }
    c->log_seq[c->log_len] = c->seq;
    c->log_row[c->log_len] = start;
    c->log_len += 1;
  }
  c->offset = start + T;
  if (c->offset > c->high_water) c->high_water = c->offset;
}

sa_status check_cache(const sa_kv_cache* c) {
  if (c == nullptr || c->k == nullptr || c->v == nullptr) return SA_ERR_INVALID_ARG;
  if (c->B < 1 || c->cap < 1 || c->n_kv < 1) return SA_ERR_INVALID_ARG;
  if (!head_dim_ok(c->d)) return SA_ERR_SHAPE;
  if (!aligned16(c->k) || !aligned16(c->v)) return SA_ERR_INVALID_ARG;
  if (c->ring < 0) return SA_ERR_INVALID_ARG;
  if (c->kv_dtype == SA_KV_FP8_E4M3) {
    if (c->k_scale == nullptr || c->v_scale == nullptr || !aligned16(c->k_scale) || !aligned16(c->v_scale))
      return SA_ERR_INVALID_ARG;
    if (c->cap % 16 != 0) return SA_ERR_SHAPE;
  } else if (c->kv_dtype != SA_KV_BF16) {
    return SA_ERR_INVALID_ARG;
  }
  if (c->ring > 0) {
    if (c->cap % kRingQuantum != 0 || c->ring > c->cap) return SA_ERR_SHAPE;
    if (c->offset < 0 || c->offset > INT32_MAX - 1) return SA_ERR_INVALID_ARG;
    return SA_OK;
  }
  if (c->offset < 0 || c->offset > c->cap) return SA_ERR_INVALID_ARG;
  return SA_OK;
}

// Checks shared by prefill and decode.
sa_status check_attn(const sa_kv_cache* c, const sa_attn_args* a) {
  sa_status st = check_cache(c);
  if (st != SA_OK) return st;
  if (a == nullptr) return SA_ERR_INVALID_ARG;
  if (a->B != c->B || a->T < 0 || a->n_q < 1) return SA_ERR_INVALID_ARG;
  if (a->n_q % c->n_kv != 0) return SA_ERR_SHAPE;
  if (a->offset != c->offset) return SA_ERR_OFFSET_MISMATCH;
  if (a->T == 0) return SA_OK;
  if (a->q == nullptr || a->k == nullptr || a->v == nullptr || a->out == nullptr)
    return SA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return SA_ERR_INVALID_ARG;
  if (!strides_ok(a->q_strides) || !strides_ok(a->k_strides) || !strides_ok(a->v_strides) ||
      !strides_ok(a->out_strides))
    return SA_ERR_INVALID_ARG;
  if (!(a->sm_scale > 0.f) || !isfinite(a->sm_scale)) return SA_ERR_INVALID_ARG;
  if (c->ring > 0) {
    if (a->window != c->ring) return SA_ERR_INVALID_ARG;
    if ((int64_t)a->T + c->ring - 1 > (int64_t)c->cap) return SA_ERR_CAPACITY;
    if (a->offset + (int64_t)a->T > (int64_t)INT32_MAX) return SA_ERR_CAPACITY;
  } else if (a->offset + (int64_t)a->T > (int64_t)c->cap) {
    return SA_ERR_CAPACITY;
  }
  if (a->rope_fused) {
    if (a->cos == nullptr || a->sin == nullptr || !aligned16(a->cos) || !aligned16(a->sin))
      return SA_ERR_INVALID_ARG;
    if (a->offset + (int64_t)a->T > (int64_t)a->max_pos) return SA_ERR_CAPACITY;
  }
  return SA_OK;
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// The shared-memory opt-in once per kernel and device (the attribute holds
// per device): `done` has one bit per device ordinal below 64, set only once
// the opt-in succeeded (a failed one is retried by the next launch, and its
// error returned); devices above 64 opt in on every call, which is harmless.
// Safe to call from several host threads (setting the attribute twice is
// harmless too).
template <typename K>
sa_status set_smem_once(K kernel, uint32_t bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return SA_OK;
  if (set_smem(kernel, bytes) != cudaSuccess) {
    cudaGetLastError();   // the failed opt-in is reported here, not by a later launch check
    return SA_ERR_CUDA;
  }
  if (bit != 0) done.fetch_or(bit, std::memory_order_release);
  return SA_OK;
}

constexpr int kMaxDevices = 64;

// Counter slots of the prefill kernel's dynamic schedule (g_prefill_sched:
// one counter pair per slot, reset by the last CTA of the launch that used
// it). Two launches in flight at once must never share a slot.
//  * Launches made outside stream capture take slots [0, kEagerSchedSlots)
//    round robin. Before one reuses a slot its stream waits for the event
//    recorded after the slot's previous launch, so the two are ordered
//    whatever streams they run on (normally that launch finished long ago
//    and the wait costs nothing).
//  * Launches captured into a CUDA graph cannot wait on work outside the
//    capture; they take slots [kEagerSchedSlots, kPrefillSchedSlots) round
//    robin, so a graph never shares a slot with an eager launch. Graph
//    replays that overlap one another must not hold more than
//    kGraphSchedSlots prefill launches between them.
constexpr int kEagerSchedSlots = sa::kPrefillSchedSlots / 2;
constexpr int kGraphSchedSlots = sa::kPrefillSchedSlots - kEagerSchedSlots;

int sched_slot_of(uint64_t index, bool captured) {
  return captured ? kEagerSchedSlots + (int)(index % kGraphSchedSlots) : (int)(index % kEagerSchedSlots);
}

struct SchedState {
  std::mutex mu;
  uint64_t eager_next = 0, graph_next = 0;
  cudaEvent_t done[kEagerSchedSlots] = {};
};
SchedState g_sched[kMaxDevices];

// Runs launch(slot) with a schedule slot acquired as above; the slot counts
// as used only if the launch succeeded.
template <typename F>
sa_status with_sched_slot(cudaStream_t s, F&& launch) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SA_ERR_INVALID_ARG;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return SA_ERR_CUDA;
  SchedState& st = g_sched[dev];
  std::lock_guard<std::mutex> lock(st.mu);
  if (cs != cudaStreamCaptureStatusNone) {
    const sa_status r = launch(sched_slot_of(st.graph_next, true));
    if (r == SA_OK) ++st.graph_next;
    return r;
  }
  const int slot = sched_slot_of(st.eager_next, false);
  cudaEvent_t& ev = st.done[slot];
  if (ev == nullptr) {
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return SA_ERR_CUDA;
  } else if (cudaStreamWaitEvent(s, ev, 0) != cudaSuccess) {
    return SA_ERR_CUDA;
  }
  const sa_status r = launch(slot);
  if (r != SA_OK) return r;
  if (cudaEventRecord(ev, s) != cudaSuccess) return SA_ERR_CUDA;
  ++st.eager_next;
  return SA_OK;
}

template <int D>
sa_status launch_prefill(const sa_kv_cache* c, const sa_attn_args* a, int slot, cudaStream_t stream) {
  using Cfg = PrefillCfg<D>;
  CUtensorMap tmQ, tmK, tmV;
  // a ring exposes all of its rows (positions outside the band are masked)
  const long long rows = c->ring > 0 ? (long long)c->cap : a->offset + a->T;
  // Query tiles come from the staged (rotated) copy in `out` when RoPE is
  // fused, else straight from q; the kernel overwrites each staged tile with
  // its output rows only after it has read it.
  const void* qsrc = a->rope_fused ? a->out : a->q;
  const int64_t* qst = a->rope_fused ? a->out_strides : a->q_strides;
  if (!make_rows_map(&tmQ, qsrc, D, a->T, a->n_q, a->B, qst, Cfg::CB)) return SA_ERR_CUDA;
  CUtensorMap tmO;   // the output tiles are stored through the same box shape
  if (!make_rows_map(&tmO, a->out, D, a->T, a->n_q, a->B, a->out_strides, Cfg::CB)) return SA_ERR_CUDA;
  // The box is one BN-row K/V tile: the kernel's expect-tx byte count and
  // ring-slot size are both Cfg::KV_BYTES = BN * D * 2.
  static_assert(Cfg::KV_BYTES == (uint32_t)Cfg::BN * D * 2, "tile size");
  if (!make_cache_map(&tmK, c->k, D, c->n_kv, rows, c->cap, c->B, Cfg::BN, Cfg::CB) ||
      !make_cache_map(&tmV, c->v, D, c->n_kv, rows, c->cap, c->B, Cfg::BN, Cfg::CB))
    return SA_ERR_CUDA;
  PrefillParams p;
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.qs0 = a->q_strides[0];
  p.qs1 = a->q_strides[1];
  p.qs2 = a->q_strides[2];
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.os0 = a->out_strides[0];
  p.os1 = a->out_strides[1];
  p.os2 = a->out_strides[2];
  p.lse = a->lse;
  p.sinks = a->sinks;
  p.cos_t = a->cos;
  p.sin_t = a->sin;
  p.B = a->B;
  p.T = a->T;
  p.n_q = a->n_q;
  p.n_kv = c->n_kv;
  p.q_mult = a->n_q / c->n_kv;
  p.off = a->offset;
  p.window = a->window > 0 ? a->window : 0;
  p.scale_log2 = a->sm_scale * 1.4426950408889634f;
  p.rope = a->rope_fused ? 1 : 0;
  p.n_pairs = (a->T + 255) / 256;
  p.ring_cap = c->ring > 0 ? c->cap : 0;
  static std::atomic<uint64_t> smem_set{0};
  {
    const sa_status sm = set_smem_once(sa::prefill_kernel<D>, Cfg::SMEM_BYTES, smem_set);
    if (sm != SA_OK) return sm;
  }
  // persistent: one CTA per SM (or per item when there are fewer)
  const long long n_items = (long long)p.n_pairs * a->n_q * a->B;
  const int grid = (int)(n_items < num_sms() ? n_items : num_sms());
  p.sched_slot = slot;
  // Programmatic stream serialization: the kernel's set-up overlaps the tail
  // of the staging launch before it; it waits for that launch to complete
  // before its first global access.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(Cfg::NUM_THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = stream;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&lc, sa::prefill_kernel<D>, tmQ, tmK, tmV, tmO, p);
  return (last_launch_status() == SA_OK && e == cudaSuccess) ? SA_OK : SA_ERR_CUDA;
}

// Band layers whose key window fits the packed-head kernel: d = 64, a
// window, q_mult dividing 128, and R + W - 1 keys (plus the 16-alignment of
// the window start) within its 160 columns (W up to 130, 114, 82 or 18 for
// q_mult 8, 4, 2 or 1). Returns the window width N (a multiple of 32) or 0.
int band_columns(const sa_kv_cache* c, const sa_attn_args* a) {
  if (c->d != 64 || a->window <= 0 || c->kv_dtype != SA_KV_BF16) return 0;
  const int qm = a->n_q / c->n_kv;
  if (qm < 1 || 128 % qm != 0) return 0;
  const long long need = 128 / qm + (long long)a->window + 14;
  const int N = (int)((need + 31) / 32 * 32);
  return N <= sa::BandCfg<64>::NMAX ? N : 0;
}

sa_status launch_band(const sa_kv_cache* c, const sa_attn_args* a, int N, cudaStream_t stream) {
  using Cfg = sa::BandCfg<64>;
  const int qm = a->n_q / c->n_kv;
  const int R = 128 / qm;
  CUtensorMap tmQ, tmK, tmV, tmKw, tmVw, tmO;
  const long long rows = c->ring > 0 ? (long long)c->cap : a->offset + a->T;
  // K/V boxes: a whole N-row window, or 16 rows (windows that wrap a ring)
  if (!make_heads_map(&tmQ, a->q, 64, a->T, a->n_q, a->B, a->q_strides, qm, R) ||
      !make_heads_map(&tmO, a->out, 64, a->T, a->n_q, a->B, a->out_strides, qm, R) ||
      !make_cache_map(&tmK, c->k, 64, c->n_kv, rows, c->cap, c->B, 16, 64) ||
      !make_cache_map(&tmV, c->v, 64, c->n_kv, rows, c->cap, c->B, 16, 64) ||
      !make_cache_map(&tmKw, c->k, 64, c->n_kv, rows, c->cap, c->B, N, 64) ||
      !make_cache_map(&tmVw, c->v, 64, c->n_kv, rows, c->cap, c->B, N, 64))
    return SA_ERR_CUDA;
  sa::BandParams p;
  p.lse = a->lse;
  p.sinks = a->sinks;
  p.cos_t = a->cos;
  p.sin_t = a->sin;
  p.B = a->B;
  p.T = a->T;
  p.n_q = a->n_q;
  p.n_kv = c->n_kv;
  p.q_mult = qm;
  p.off = a->offset;
  p.window = a->window;
  p.scale_log2 = a->sm_scale * 1.4426950408889634f;
  p.rope = a->rope_fused ? 1 : 0;
  p.ring_cap = c->ring > 0 ? c->cap : 0;
  p.R = R;
  p.N = N;
  p.n_blk = (a->T + R - 1) / R;
  const long long units = (long long)a->B * c->n_kv * p.n_blk;
  if (units > INT32_MAX) return SA_ERR_SHAPE;
  p.n_units = (int)units;
  static std::atomic<uint64_t> smem_set{0};
  {
    const sa_status sm = set_smem_once(sa::band_kernel<64>, Cfg::SMEM_BYTES, smem_set);
    if (sm != SA_OK) return sm;
  }
  // persistent: one CTA per SM (or per unit when there are fewer)
  const int grid = (int)(units < num_sms() ? units : num_sms());
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(Cfg::NUM_THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = stream;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&lc, sa::band_kernel<64>, tmQ, tmK, tmV, tmKw, tmVw, tmO, p);
  return (last_launch_status() == SA_OK && e == cudaSuccess) ? SA_OK : SA_ERR_CUDA;
}

// CTAs per (b, g) for n_cache cached rows in stages of `stage` rows: at
// most one wave of CTAs (two per SM) -- the decode kernel balances the
// stages among the CTAs of each (b, g) by itself, and a partial second wave
// would only stream its CTAs' static stages at the end -- and no more CTAs
// than stages.
int decode_splits(int B, int n_kv, long long n_cache, long long stage) {
  if (n_cache <= 0) return 1;
  long long S = 2LL * num_sms() / ((long long)B * n_kv);
  const long long nb = (n_cache + stage - 1) / stage;
  if (S > nb) S = nb;
  return S < 1 ? 1 : (int)S;
}

// Workspace layout: split tickets [B*n_kv] then dynamic-stage counters
// [B*n_kv], int32 (256-byte padded), then one fp32 record per (b, g, split):
// O [q_mult][d], m [q_mult], l [q_mult], padded to a multiple of 16 bytes
// (the merge brings records in by bulk copy).
int decode_rec_floats(int q_mult, int d) { return q_mult * d + (2 * q_mult + 3) / 4 * 4; }

size_t decode_cnt_bytes(int B, int n_kv) { return (((size_t)B * n_kv * 8) + 255) / 256 * 256; }

size_t decode_ws_bytes(int B, int n_kv, int q_mult, int d, int S) {
  return decode_cnt_bytes(B, n_kv) + (size_t)B * n_kv * S * decode_rec_floats(q_mult, d) * 4;
}

// Cache rows per ring stage of decode_kernel<d, f8> (its Cfg::R).
long long decode_stage_rows(int d, bool f8) {
  switch (d) {
    case 64: return f8 ? sa::DecodeCfgT<64, true>::R : sa::DecodeCfgT<64, false>::R;
    case 96: return f8 ? sa::DecodeCfgT<96, true>::R : sa::DecodeCfgT<96, false>::R;
    default: return f8 ? sa::DecodeCfgT<128, true>::R : sa::DecodeCfgT<128, false>::R;
  }
}

// The rows one decode call reads and how they are split over CTAs: the
// launch and the allocation-free entry point's size check both take it from
// here. lo_mask: first admitted key; lo: first row streamed (ring and FP8
// stages start on multiples of the stage height, so no TMA box wraps a ring
// and the scale boxes start on their stage's first row).
struct DecodePlan {
  long long lo_mask, lo;
  int S;   // CTAs per (b, g)
};

DecodePlan plan_decode(const sa_kv_cache* c, const sa_attn_args* a) {
  const bool f8 = c->kv_dtype == SA_KV_FP8_E4M3;
  const long long R = decode_stage_rows(c->d, f8);
  DecodePlan pl;
  pl.lo_mask = a->window > 0 ? (a->offset + 1 - a->window > 0 ? a->offset + 1 - a->window : 0) : 0;
  pl.lo = (c->ring > 0 || f8) ? pl.lo_mask / R * R : pl.lo_mask;
  pl.S = decode_splits(a->B, c->n_kv, a->offset - pl.lo, R);
  return pl;
}

// Cache bytes each decode CTA prefetches into L2 before it waits for the
// kernel ahead of it on the stream (rounded up to whole stages).
constexpr long long kDecodePrefetchBytes = 128 * 1024;

template <int D, bool F8>
sa_status launch_decode(const sa_kv_cache* c, const sa_attn_args* a, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
  using Cfg = sa::DecodeCfgT<D, F8>;
  const int q_mult = a->n_q / c->n_kv;
  DecodeParams p;
  p.off = a->offset;
  p.ring_cap = c->ring > 0 ? c->cap : 0;
  const DecodePlan pl = plan_decode(c, a);
  p.lo_mask = pl.lo_mask;
  p.lo = pl.lo;
  const long long n_cache = p.off - p.lo;
  p.S = pl.S;
  p.n_blocks = n_cache > 0 ? (n_cache + Cfg::R - 1) / Cfg::R : 0;
  // a lone CTA streams everything in order; with several, half of each
  // one's share is static and the rest dynamic
  p.static_stages = p.S == 1 ? (int)p.n_blocks : (int)(p.n_blocks / (2 * p.S));
  p.pf_stages = (int)((kDecodePrefetchBytes + Cfg::STAGE_TX - 1) / Cfg::STAGE_TX);
  if (p.S > 1) {
    if (ws == nullptr || !aligned16(ws) || ws_bytes < decode_ws_bytes(a->B, c->n_kv, q_mult, D, p.S))
      return SA_ERR_WORKSPACE;
  }
  CUtensorMap tmK, tmV, tmKS, tmVS;
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  memset(&tmKS, 0, sizeof(tmKS));
  memset(&tmVS, 0, sizeof(tmVS));
  if (n_cache > 0) {
    const long long rows = p.ring_cap > 0 ? (long long)c->cap : p.off;
    constexpr int kBoxRows = Cfg::R / Cfg::NBOX;   // a stage is NBOX boxes of 128 rows
    static_assert(kBoxRows == 128, "decode TMA boxes are 128 rows");
    if constexpr (F8) {
      if (!make_codes_map(&tmK, c->k, D, c->n_kv, rows, c->cap, c->B, kBoxRows, Cfg::ROWB) ||
          !make_codes_map(&tmV, c->v, D, c->n_kv, rows, c->cap, c->B, kBoxRows, Cfg::ROWB) ||
          !make_scales_map(&tmKS, c->k_scale, c->n_kv, rows, c->cap, c->B, kBoxRows) ||
          !make_scales_map(&tmVS, c->v_scale, c->n_kv, rows, c->cap, c->B, kBoxRows))
        return SA_ERR_CUDA;
    } else {
      if (!make_cache_map(&tmK, c->k, D, c->n_kv, rows, c->cap, c->B, kBoxRows, Cfg::CB) ||
          !make_cache_map(&tmV, c->v, D, c->n_kv, rows, c->cap, c->B, kBoxRows, Cfg::CB))
        return SA_ERR_CUDA;
    }
  }
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.qs0 = a->q_strides[0];
  p.qs2 = a->q_strides[2];
  p.k = static_cast<const __nv_bfloat16*>(a->k);
  p.ks0 = a->k_strides[0];
  p.ks2 = a->k_strides[2];
  p.v = static_cast<const __nv_bfloat16*>(a->v);
  p.vs0 = a->v_strides[0];
  p.vs2 = a->v_strides[2];
  p.ck = static_cast<__nv_bfloat16*>(c->k);
  p.cv = static_cast<__nv_bfloat16*>(c->v);
  p.cap = c->cap;
  p.cks = static_cast<float*>(c->k_scale);
  p.cvs = static_cast<float*>(c->v_scale);
  p.out = static_cast<__nv_bfloat16*>(a->out);
  p.os0 = a->out_strides[0];
  p.os2 = a->out_strides[2];
  p.lse = a->lse;
  p.sinks = a->sinks;
  p.cos_t = a->cos;
  p.sin_t = a->sin;
  p.B = a->B;
  p.n_q = a->n_q;
  p.n_kv = c->n_kv;
  p.q_mult = q_mult;
  p.scale_log2 = a->sm_scale * 1.4426950408889634f;
  p.rope = a->rope_fused ? 1 : 0;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ws_cnt = reinterpret_cast<int*>(w);
  p.ws_grab = p.ws_cnt + (size_t)a->B * c->n_kv;
  p.ws_rec = reinterpret_cast<float*>(w + decode_cnt_bytes(a->B, c->n_kv));
  p.rec_floats = decode_rec_floats(q_mult, D);
  static std::atomic<uint64_t> smem_set{0};
  {
    const sa_status sm = set_smem_once(sa::decode_kernel<D, F8>, Cfg::SMEM_BYTES, smem_set);
    if (sm != SA_OK) return sm;
  }
  // Programmatic stream serialization: back-to-back decode launches (one per
  // layer) overlap one kernel's drain with the next one's launch and set-up;
  // the kernel waits for its predecessor before touching global memory.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(c->n_kv, p.S, a->B);
  lc.blockDim = dim3(Cfg::NUM_THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = stream;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&lc, sa::decode_kernel<D, F8>, tmK, tmV, tmKS, tmVS, p);
  return (last_launch_status() == SA_OK && e == cudaSuccess) ? SA_OK : SA_ERR_CUDA;
}

sa_status launch_append(sa_kv_cache* c, const void* k, const int64_t ks[3], const void* v,
                        const int64_t vs[3], int T, int rope, const float* cos_t,
                        const float* sin_t, cudaStream_t stream) {
  if (c->kv_dtype == SA_KV_FP8_E4M3) {
    if (rope) return SA_ERR_UNSUPPORTED;
    const long long rows = (long long)c->B * T * c->n_kv;   // one warp per row
    sa::kv_append_fp8_kernel<<<grid_for(rows * 32), 256, 0, stream>>>(
        static_cast<uint8_t*>(c->k), static_cast<uint8_t*>(c->v), static_cast<float*>(c->k_scale),
        static_cast<float*>(c->v_scale), c->cap, static_cast<const __nv_bfloat16*>(k), ks[0], ks[1],
        ks[2], static_cast<const __nv_bfloat16*>(v), vs[0], vs[1], vs[2], c->B, T, c->n_kv, c->d,
        c->offset, c->ring > 0 ? 1 : 0);
    return last_launch_status();
  }
  const long long n = (long long)c->B * T * c->n_kv * (c->d / 16);
  sa::kv_append_kernel<<<grid_for(n), 256, 0, stream>>>(
      static_cast<__nv_bfloat16*>(c->k), static_cast<__nv_bfloat16*>(c->v), c->cap,
      static_cast<const __nv_bfloat16*>(k), ks[0], ks[1], ks[2],
      static_cast<const __nv_bfloat16*>(v), vs[0], vs[1], vs[2], c->B, T, c->n_kv, c->d, c->offset,
      rope, cos_t, sin_t, c->ring > 0 ? 1 : 0);
  return last_launch_status();
}

// Events of sa_set_prefill_events (null: not recording).
cudaEvent_t g_prefill_ev_before = nullptr;
cudaEvent_t g_prefill_ev_after = nullptr;

// Prefill staging, one launch: append K/V (rotating k when RoPE is fused)
// and, with stage_q, write the rotated queries into `out` for the attention
// kernel to load by TMA.
sa_status launch_stage(sa_kv_cache* c, const sa_attn_args* a, bool stage_q, cudaStream_t stream) {
  const long long n = (long long)c->B * a->T * (c->n_kv + (stage_q ? a->n_q : 0)) * (c->d / 16);
  sa::prefill_stage_kernel<<<grid_for(n), 256, 0, stream>>>(
      static_cast<__nv_bfloat16*>(c->k), static_cast<__nv_bfloat16*>(c->v), c->cap,
      static_cast<const __nv_bfloat16*>(a->k), a->k_strides[0], a->k_strides[1], a->k_strides[2],
      static_cast<const __nv_bfloat16*>(a->v), a->v_strides[0], a->v_strides[1], a->v_strides[2],
      c->B, a->T, c->n_kv, c->d, c->offset, a->rope_fused ? 1 : 0, a->cos, a->sin,
      static_cast<const __nv_bfloat16*>(a->q), a->q_strides[0], a->q_strides[1], a->q_strides[2],
      a->n_q, static_cast<__nv_bfloat16*>(a->out), a->out_strides[0], a->out_strides[1],
      a->out_strides[2], stage_q ? 1 : 0, c->ring > 0 ? 1 : 0);
  return last_launch_status();
}

// Scratch of sa_attn_decode_static: one fixed array per device, its device
// address looked up once per device (host code may not use the symbol itself
// as an address).
static __device__ __align__(256) uint8_t g_decode_scratch[SA_DECODE_STATIC_SCRATCH_BYTES];
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

sa_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) return SA_ERR_CUDA;
    // the split counters must start at zero (each call leaves them at zero)
    if (cudaMemset(ptr, 0, SA_DECODE_STATIC_SCRATCH_BYTES) != cudaSuccess) return SA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return SA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

// Projections around the attention: one GEMM launch (csrc/gemm.cuh).

bool matrix_ok(const void* p, int64_t ld, int64_t cols) {
  return p != nullptr && aligned16(p) && ld >= cols && ld % 8 == 0;
}

template <int BN>
sa_status launch_gemm_bn(const void* a, int64_t lda, const void* w, int64_t ldw, const void* bias,
                         const void* residual, int64_t ldr, void* y, int64_t ldy, int32_t M, int32_t N,
                         int32_t K, int rms, float eps, cudaStream_t stream) {
  using C = sa::GemmCfg<BN>;
  CUtensorMap tmA, tmB, tmC;
  if (!make_matrix_map(&tmA, a, K, M, lda, C::BK, C::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_matrix_map(&tmB, w, K, N, ldw, C::BK, C::BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_matrix_map(&tmC, y, N, M, ldy, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return SA_ERR_CUDA;
  sa::GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.residual = static_cast<const __nv_bfloat16*>(residual);
  p.ldr = ldr;
  p.rms = rms;
  p.eps = eps;
  p.tiles_m = (M + C::BM - 1) / C::BM;
  p.tiles_n = (N + C::BN - 1) / C::BN;
  const long long tiles = (long long)p.tiles_m * p.tiles_n;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  static std::atomic<uint64_t> smem_set{0};
  {
    const sa_status sm = set_smem_once(sa::gemm_kernel<BN>, C::SMEM_BYTES, smem_set);
    if (sm != SA_OK) return sm;
  }
  sa::gemm_kernel<BN><<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(tmA, tmB, tmC, p);
  return last_launch_status();
}

// 256 x 256 tiles. Narrower tiles fill the last wave of tiles better but
// measured slower on the gpt-oss qkv projection (4.3 waves of 256-column
// tiles): 160 columns 254 us, 192 columns 226 us, 256 columns 197-200 us.
sa_status launch_gemm(const void* a, int64_t lda, const void* w, int64_t ldw, const void* bias,
                      const void* residual, int64_t ldr, void* y, int64_t ldy, int32_t M, int32_t N,
                      int32_t K, int rms, float eps, cudaStream_t stream) {
  return launch_gemm_bn<256>(a, lda, w, ldw, bias, residual, ldr, y, ldy, M, N, K, rms, eps, stream);
}

// Backward pass (csrc/backward.cuh): the row pass, then one launch of the
// products (csrc/backward_tc.cuh).
template <int D>
sa_status launch_backward(const sa_attn_bwd_args* a, float* dvec, cudaStream_t stream) {
  sa::BwdParams p;
  p.q = static_cast<const __nv_bfloat16*>(a->q);
  p.k = static_cast<const __nv_bfloat16*>(a->k);
  p.v = static_cast<const __nv_bfloat16*>(a->v);
  p.o = static_cast<const __nv_bfloat16*>(a->out);
  p.dout = static_cast<const __nv_bfloat16*>(a->d_out);
  p.qs0 = a->q_strides[0]; p.qs1 = a->q_strides[1]; p.qs2 = a->q_strides[2];
  p.ks0 = a->k_strides[0]; p.ks1 = a->k_strides[1]; p.ks2 = a->k_strides[2];
  p.vs0 = a->v_strides[0]; p.vs1 = a->v_strides[1]; p.vs2 = a->v_strides[2];
  p.os0 = a->out_strides[0]; p.os1 = a->out_strides[1]; p.os2 = a->out_strides[2];
  p.ds0 = a->d_out_strides[0]; p.ds1 = a->d_out_strides[1]; p.ds2 = a->d_out_strides[2];
  p.lse = a->lse;
  p.sinks = a->sinks;
  // rows padded to a multiple of 384 (every streamed tile's 64, 96 or 128
  // values lie inside its row; 16-byte aligned)
  p.Tp = bwd_rows_padded(a->T);
  p.dvec = dvec;
  p.lse2 = dvec + (size_t)a->B * a->n_q * p.Tp;
  p.dq = a->dq;
  p.dk = a->dk;
  p.dv = a->dv;
  p.dsinks = a->sinks ? a->dsinks : nullptr;
  p.B = a->B;
  p.T = a->T;
  p.n_q = a->n_q;
  p.n_kv = a->n_kv;
  p.q_mult = a->n_q / a->n_kv;
  p.window = a->window;
  p.scale = a->sm_scale;
  p.scale_log2 = a->sm_scale * 1.4426950408889634f;
  if (p.dsinks && cudaMemsetAsync(p.dsinks, 0, sizeof(float) * a->n_q, stream) != cudaSuccess) return SA_ERR_CUDA;
  const long long rows = (long long)a->B * p.Tp * a->n_q;
  sa::bwd_rows_kernel<D><<<grid_for(rows * 4), 256, (size_t)a->n_q * sizeof(float), stream>>>(p);
  using C = sa::BkvCfg<D>;
  // resident K, V (128 rows); streamed Q, dO (BN rows)
  CUtensorMap tk, tv, tq, to, tdq;
  if (!make_rows_map(&tk, a->k, D, a->T, a->n_kv, a->B, a->k_strides, C::CB, C::BM) ||
      !make_rows_map(&tv, a->v, D, a->T, a->n_kv, a->B, a->v_strides, C::CB, C::BM) ||
      !make_rows_map(&tq, a->q, D, a->T, a->n_q, a->B, a->q_strides, C::CB, C::BN) ||
      !make_rows_map(&to, a->d_out, D, a->T, a->n_q, a->B, a->d_out_strides, C::CB, C::BN) ||
      !make_f32_rows_map(&tdq, a->dq, D, a->T, a->n_q, a->B, C::BN))
    return SA_ERR_CUDA;
  static std::atomic<uint64_t> smem_set{0};
  {
    const sa_status sm = set_smem_once(sa::bwd_tc_kernel<D>, C::SMEM_BYTES, smem_set);
    if (sm != SA_OK) return sm;
  }
  // one CTA per 128-key tile, per KV head, per sequence (< 2^31: checked by the caller)
  const unsigned ctas = (unsigned)((a->T + 127) / 128) * (unsigned)a->n_kv * (unsigned)a->B;
  sa::bwd_tc_kernel<D><<<ctas, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(tk, tv, tq, to, tdq, p);
  return last_launch_status();
}

}  // namespace

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_SHAPE: return "SA_ERR_SHAPE";
    case SA_ERR_CAPACITY: return "SA_ERR_CAPACITY";
    case SA_ERR_OFFSET_MISMATCH: return "SA_ERR_OFFSET_MISMATCH";
    case SA_ERR_STALE_SNAPSHOT: return "SA_ERR_STALE_SNAPSHOT";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
  }
  return "SA_UNKNOWN";
}

sa_status sa_yarn_rope_tables(float* cos_out, float* sin_out, int32_t max_pos, int32_t d,
                              double theta, double scaling, int32_t orig_ctx, double alpha,
                              double beta, sa_stream_t stream) {
  if (cos_out == nullptr || sin_out == nullptr || max_pos < 1 || d < 2 || d % 2 != 0)
    return SA_ERR_INVALID_ARG;
  if (!(theta > 1.0) || !(scaling > 0.0) || orig_ctx < 1 || !(alpha > 0.0) || !(beta > 0.0) ||
      !(alpha < beta))
    return SA_ERR_INVALID_ARG;
  const int half = d / 2;
  sa::yarn_tables_kernel<<<grid_for((long long)max_pos * half), 256, 0, (cudaStream_t)stream>>>(
      cos_out, sin_out, max_pos, half, theta, scaling, (double)orig_ctx, alpha, beta);
  return last_launch_status();
}

sa_status sa_rope_apply_qk(void* q, const int64_t q_strides[3], void* k, const int64_t k_strides[3],
                           int32_t B, int32_t T, int32_t n_q, int32_t n_kv, int32_t d,
                           int64_t offset, const float* cos, const float* sin, int32_t max_pos,
                           sa_stream_t stream) {
  if (B < 0 || T < 0 || n_q < 0 || n_kv < 0 || offset < 0) return SA_ERR_INVALID_ARG;
  if (!head_dim_ok(d)) return SA_ERR_SHAPE;
  if (cos == nullptr || sin == nullptr || !aligned16(cos) || !aligned16(sin)) return SA_ERR_INVALID_ARG;
  if (q != nullptr && (!aligned16(q) || !strides_ok(q_strides))) return SA_ERR_INVALID_ARG;
  if (k != nullptr && (!aligned16(k) || !strides_ok(k_strides))) return SA_ERR_INVALID_ARG;
  if (offset + (int64_t)T > (int64_t)max_pos) return SA_ERR_CAPACITY;
  if (B == 0 || T == 0) return SA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (q != nullptr && n_q > 0) {
    const long long n = (long long)B * T * n_q * (d / 16);
    sa::rope_inplace_kernel<<<grid_for(n), 256, 0, s>>>(static_cast<__nv_bfloat16*>(q), q_strides[0],
                                                        q_strides[1], q_strides[2], B, T, n_q, d,
                                                        offset, cos, sin);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  if (k != nullptr && n_kv > 0) {
    const long long n = (long long)B * T * n_kv * (d / 16);
    sa::rope_inplace_kernel<<<grid_for(n), 256, 0, s>>>(static_cast<__nv_bfloat16*>(k), k_strides[0],
                                                        k_strides[1], k_strides[2], B, T, n_kv, d,
                                                        offset, cos, sin);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

sa_status sa_kv_cache_init(sa_kv_cache* cache, void* k, void* v, int32_t B, int32_t cap,
                           int32_t n_kv, int32_t d) {
  if (cache == nullptr) return SA_ERR_INVALID_ARG;
  memset(cache, 0, sizeof(*cache));
  cache->k = k;
  cache->v = v;
  cache->B = B;
  cache->cap = cap;
  cache->n_kv = n_kv;
  cache->d = d;
  cache->log_floor_seq = -1;
  cache->log_floor_row = INT64_MAX;
  return check_cache(cache);
}

sa_status sa_kv_cache_init_ring(sa_kv_cache* cache, void* k, void* v, int32_t B, int32_t cap,
                                int32_t n_kv, int32_t d, int32_t window) {
  if (cache == nullptr || window < 1) return SA_ERR_INVALID_ARG;
  sa_status st = sa_kv_cache_init(cache, k, v, B, cap, n_kv, d);
  if (st != SA_OK) return st;
  cache->ring = window;
  return check_cache(cache);
}

sa_status sa_kv_cache_init_fp8(sa_kv_cache* cache, void* k, void* v, void* k_scale, void* v_scale,
                               int32_t B, int32_t cap, int32_t n_kv, int32_t d, int32_t window) {
  if (cache == nullptr || window < 0) return SA_ERR_INVALID_ARG;
  sa_status st = sa_kv_cache_init(cache, k, v, B, cap, n_kv, d);
  if (st != SA_OK) return st;
  cache->ring = window;
  cache->kv_dtype = SA_KV_FP8_E4M3;
  cache->k_scale = k_scale;
  cache->v_scale = v_scale;
  return check_cache(cache);
}

sa_status sa_kv_append(sa_kv_cache* cache, const void* k_rot, const int64_t k_strides[3],
                       const void* v, const int64_t v_strides[3], int32_t T, sa_stream_t stream) {
  sa_status st = check_cache(cache);
  if (st != SA_OK) return st;
  if (T < 0) return SA_ERR_INVALID_ARG;
  if (T == 0) return SA_OK;
  if (k_rot == nullptr || v == nullptr || !aligned16(k_rot) || !aligned16(v) ||
      !strides_ok(k_strides) || !strides_ok(v_strides))
    return SA_ERR_INVALID_ARG;
  if (cache->ring > 0 ? (T > cache->cap || cache->offset + (int64_t)T > (int64_t)INT32_MAX)
                      : cache->offset + (int64_t)T > (int64_t)cache->cap)
    return SA_ERR_CAPACITY;
  st = launch_append(cache, k_rot, k_strides, v, v_strides, T, 0, nullptr, nullptr,
                     (cudaStream_t)stream);
  if (st != SA_OK) return st;
  note_append(cache, cache->offset, T);
  return SA_OK;
}

sa_status sa_kv_snapshot(const sa_kv_cache* cache, sa_snapshot* out) {
  sa_status st = check_cache(cache);
  if (st != SA_OK) return st;
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  out->cache_id = (uint64_t)reinterpret_cast<uintptr_t>(cache->k);
  out->offset = cache->offset;
  out->seq = cache->seq;
  out->cap = cache->cap;
  return SA_OK;
}

sa_status sa_kv_restore(sa_kv_cache* cache, const sa_snapshot* snap) {
  sa_status st = check_cache(cache);
  if (st != SA_OK) return st;
  if (snap == nullptr) return SA_ERR_INVALID_ARG;
  if (snap->cache_id != (uint64_t)reinterpret_cast<uintptr_t>(cache->k) || snap->cap != cache->cap ||
      snap->offset < 0 || snap->offset > cache->high_water || snap->seq > cache->seq)
    return SA_ERR_INVALID_ARG;
  if (snap->seq < cache->log_floor_seq && cache->log_floor_row < snap->offset) return SA_ERR_STALE_SNAPSHOT;
  // a ring keeps the last cap positions: the band rows the snapshot needs,
  // [offset - ring + 1, offset), must not have been overwritten since
  if (cache->ring > 0 && cache->high_water > snap->offset + cache->cap - (cache->ring - 1))
    return SA_ERR_STALE_SNAPSHOT;
  for (int i = 0; i < cache->log_len; ++i)
    if (cache->log_seq[i] > snap->seq && cache->log_row[i] < snap->offset) return SA_ERR_STALE_SNAPSHOT;
  cache->offset = snap->offset;
  cache->seq += 1;
  return SA_OK;
}

sa_status sa_attn_prefill(sa_kv_cache* cache, const sa_attn_args* a, sa_stream_t stream) {
  sa_status st = check_attn(cache, a);
  if (st != SA_OK) return st;
  if (cache->kv_dtype != SA_KV_BF16) return SA_ERR_UNSUPPORTED;
  if (a->T == 0) return SA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  bool staged = false;
  const int band_n = band_columns(cache, a);
  if (band_n > 0) {
    // band layer with packed heads: the staging launch appends K/V only (the
    // kernel rotates its own queries) and the kernel needs no schedule slot
    st = launch_stage(cache, a, false, s);
    if (st == SA_OK) {
      staged = true;
      cudaEvent_t ev0 = g_prefill_ev_before, ev1 = g_prefill_ev_after;
      if (ev0 != nullptr && cudaEventRecord(ev0, s) != cudaSuccess) st = SA_ERR_CUDA;
      if (st == SA_OK) st = launch_band(cache, a, band_n, s);
      if (st == SA_OK && ev1 != nullptr && cudaEventRecord(ev1, s) != cudaSuccess) st = SA_ERR_CUDA;
    }
    if (staged) note_append(cache, cache->offset, a->T);
    return st;
  }
  // The schedule slot (and the wait for its previous user) is taken before
  // the staging launch, so nothing stands between the two kernels.
  st = with_sched_slot(s, [&](int slot) -> sa_status {
    // one launch: the call's K rows rotated (when RoPE is fused) and appended
    // with V, and the rotated queries staged in `out`
    sa_status r = launch_stage(cache, a, a->rope_fused, s);
    if (r != SA_OK) return r;
    staged = true;
    cudaEvent_t ev0 = g_prefill_ev_before, ev1 = g_prefill_ev_after;
    if (ev0 != nullptr && cudaEventRecord(ev0, s) != cudaSuccess) return SA_ERR_CUDA;
    switch (cache->d) {
      case 64: r = launch_prefill<64>(cache, a, slot, s); break;
      case 96: r = launch_prefill<96>(cache, a, slot, s); break;
      default: r = launch_prefill<128>(cache, a, slot, s); break;
    }
    if (ev1 != nullptr && cudaEventRecord(ev1, s) != cudaSuccess) return SA_ERR_CUDA;
    return r;
  });
  // Once the append is enqueued the offset follows it.
  if (staged) note_append(cache, cache->offset, a->T);
  return st;
}

sa_status sa_attn_decode(sa_kv_cache* cache, const sa_attn_args* a, void* workspace,
                         size_t workspace_bytes, sa_stream_t stream) {
  sa_status st = check_attn(cache, a);
  if (st != SA_OK) return st;
  if (a->T != 1) return SA_ERR_INVALID_ARG;
  if (a->n_q / cache->n_kv > 8) return SA_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  const bool f8 = cache->kv_dtype == SA_KV_FP8_E4M3;
  switch (cache->d) {
    case 64:
      st = f8 ? launch_decode<64, true>(cache, a, workspace, workspace_bytes, s)
              : launch_decode<64, false>(cache, a, workspace, workspace_bytes, s);
      break;
    case 96:
      st = f8 ? launch_decode<96, true>(cache, a, workspace, workspace_bytes, s)
              : launch_decode<96, false>(cache, a, workspace, workspace_bytes, s);
      break;
    case 128:
      st = f8 ? launch_decode<128, true>(cache, a, workspace, workspace_bytes, s)
              : launch_decode<128, false>(cache, a, workspace, workspace_bytes, s);
      break;
    default: return SA_ERR_SHAPE;
  }
  if (st == SA_OK) note_append(cache, cache->offset, 1);
  return st;
}

sa_status sa_attn_decode_static(sa_kv_cache* cache, const sa_attn_args* a, sa_stream_t stream) {
  sa_status st = check_attn(cache, a);
  if (st != SA_OK) return st;
  if (a->T != 1) return SA_ERR_INVALID_ARG;
  const int q_mult = a->n_q / cache->n_kv;
  if (q_mult > 8) return SA_ERR_SHAPE;
  const int S = plan_decode(cache, a).S;   // the split the launch will use
  if (S > 1 && decode_ws_bytes(a->B, cache->n_kv, q_mult, cache->d, S) > SA_DECODE_STATIC_SCRATCH_BYTES)
    return SA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != SA_OK) return st;
  return sa_attn_decode(cache, a, scratch, SA_DECODE_STATIC_SCRATCH_BYTES, stream);
}

size_t sa_attn_decode_workspace_size(int32_t B, int32_t n_q, int32_t n_kv, int32_t d) {
  if (B < 1 || n_kv < 1 || n_q < n_kv || d < 1) return 0;
  const int q_mult = n_q / n_kv;
  // B*n_kv*S <= 2*256 + B*n_kv for any device of at most 256 SMs.
  const long long units = 512 + (long long)B * n_kv;
  return decode_cnt_bytes(B, n_kv) + (size_t)units * decode_rec_floats(q_mult, d) * 4;
}

sa_status sa_rmsnorm_fold_weight(const void* w, int64_t ldw, const float* gamma, void* w_folded,
                                 int64_t ldf, int32_t N, int32_t K, sa_stream_t stream) {
  if (N < 1 || K < 1 || gamma == nullptr || !matrix_ok(w, ldw, K) || !matrix_ok(w_folded, ldf, K))
    return SA_ERR_INVALID_ARG;
  sa::fold_gamma_kernel<<<grid_for((long long)N * K), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const __nv_bfloat16*>(w), ldw, gamma, static_cast<__nv_bfloat16*>(w_folded), ldf, N, K);
  return last_launch_status();
}

sa_status sa_qkv_proj(const void* x, int64_t ldx, const void* w_folded, int64_t ldw, const void* bias,
                      float eps, void* y, int64_t ldy, int32_t M, int32_t N, int32_t K, sa_stream_t stream) {
  if (M < 0 || N < 1 || K < 1 || !(eps >= 0.f) || !isfinite(eps)) return SA_ERR_INVALID_ARG;
  if (M == 0) return SA_OK;
  if (!matrix_ok(x, ldx, K) || !matrix_ok(w_folded, ldw, K) || !matrix_ok(y, ldy, N) ||
      (bias != nullptr && !aligned16(bias)))
    return SA_ERR_INVALID_ARG;
  return launch_gemm(x, ldx, w_folded, ldw, bias, nullptr, 0, y, ldy, M, N, K, 1, eps, (cudaStream_t)stream);
}

sa_status sa_out_proj(const void* o, int64_t ldo, const void* w, int64_t ldw, const void* bias, void* x,
                      int64_t ldx, int32_t M, int32_t N, int32_t K, sa_stream_t stream) {
  if (M < 0 || N < 1 || K < 1) return SA_ERR_INVALID_ARG;
  if (M == 0) return SA_OK;
  if (!matrix_ok(o, ldo, K) || !matrix_ok(w, ldw, K) || !matrix_ok(x, ldx, N) ||
      (bias != nullptr && !aligned16(bias)))
    return SA_ERR_INVALID_ARG;
  return launch_gemm(o, ldo, w, ldw, bias, x, ldx, x, ldx, M, N, K, 0, 0.f, (cudaStream_t)stream);
}

size_t sa_attn_backward_workspace_size(int32_t B, int32_t T, int32_t n_q) {
  if (B < 1 || T < 1 || n_q < 1) return 0;
  const size_t Tp = (size_t)bwd_rows_padded(T);   // D and lse * log2(e), rows padded to 384 entries
  return (2 * (size_t)B * n_q * Tp * 4 + 255) / 256 * 256;
}

sa_status sa_attn_backward(const sa_attn_bwd_args* a, void* workspace, size_t workspace_bytes,
                           sa_stream_t stream) {
  if (a == nullptr || a->B < 1 || a->T < 1 || a->n_q < 1 || a->n_kv < 1) return SA_ERR_INVALID_ARG;
  if (!head_dim_ok(a->d)) return SA_ERR_SHAPE;
  if (a->n_q % a->n_kv != 0) return SA_ERR_SHAPE;
  // the row pass sums n_q floats in shared memory; the products launch one CTA
  // per 128-key tile, per KV head, per sequence (a 1-D grid)
  const long long ctas = (long long)((a->T + 127) / 128) * a->n_kv * a->B;
  if (a->n_q > 8192 || ctas > 0x7fffffffLL) return SA_ERR_SHAPE;
  const void* ins[5] = {a->q, a->k, a->v, a->out, a->d_out};
  const int64_t* st[5] = {a->q_strides, a->k_strides, a->v_strides, a->out_strides, a->d_out_strides};
  for (int i = 0; i < 5; ++i)
    if (ins[i] == nullptr || !aligned16(ins[i]) || !strides_ok(st[i])) return SA_ERR_INVALID_ARG;
  if (a->lse == nullptr || a->dq == nullptr || a->dk == nullptr || a->dv == nullptr) return SA_ERR_INVALID_ARG;
  if (!aligned16(a->dq) || !aligned16(a->dk) || !aligned16(a->dv)) return SA_ERR_INVALID_ARG;
  if (!(a->sm_scale > 0.f) || !isfinite(a->sm_scale)) return SA_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace) ||
      workspace_bytes < sa_attn_backward_workspace_size(a->B, a->T, a->n_q))
    return SA_ERR_WORKSPACE;
  float* dvec = static_cast<float*>(workspace);
  cudaStream_t s = (cudaStream_t)stream;
  switch (a->d) {
    case 64: return launch_backward<64>(a, dvec, s);
    case 96: return launch_backward<96>(a, dvec, s);
    case 128: return launch_backward<128>(a, dvec, s);
  }
  return SA_ERR_SHAPE;
}

sa_status sa_get_device_status(int32_t* code) {
  if (code == nullptr) return SA_ERR_INVALID_ARG;
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return SA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, sa::g_status, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(sa::g_status, &zero, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
  *code = (v & sa::STATUS_TIMEOUT) ? SA_ERR_TIMEOUT : SA_OK;
  return SA_OK;
}

sa_status sa_set_prefill_events(void* before, void* after) {
  if ((before == nullptr) != (after == nullptr)) return SA_ERR_INVALID_ARG;
  g_prefill_ev_before = static_cast<cudaEvent_t>(before);
  g_prefill_ev_after = static_cast<cudaEvent_t>(after);
  return SA_OK;
}

int32_t sa_prefill_sched_slot(uint64_t index, int32_t captured) {
  return sched_slot_of(index, captured != 0);
}

sa_status sa_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return SA_ERR_INVALID_ARG;
  long long v = cycles;
  if (cudaMemcpyToSymbol(sa::g_wait_limit, &v, sizeof(v)) != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

}  // extern "C"
