/*
 * libsinkattn -- gpt-oss-style sink-augmented grouped-query attention for
 * NVIDIA B200 (sm_100a). Plain C ABI: pointers, sizes and status codes only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - bf16 tensors are passed as void pointers to 16-bit bfloat16 storage.
 * - "Device" pointers must be CUDA device memory of the current device;
 *   "host" pointers are ordinary host memory.
 * - Strides are in ELEMENTS. A q/k/v/out operand of logical shape
 *   [B][T][H][d] is addressed as base + b*s[0] + t*s[1] + h*s[2] + c, i.e.
 *   the last (head-width) dimension must be contiguous. This admits views
 *   into a fused qkv tensor [B][T][d*(n_q+2*n_kv)] (GQA Attention study note,
 *   "How it works": the fused qkv width 5120 split into Q, K, V).
 *   Every base pointer and stride must keep 16-byte alignment of each row
 *   (d*2 bytes rows, strides multiples of 8 elements).
 * - All device work is enqueued asynchronously on the given stream (NULL =
 *   the legacy default stream). Argument checks run on the host BEFORE any
 *   launch: a call that returns an error other than SA_ERR_CUDA has enqueued
 *   nothing and changed no state.
 * - The library never allocates device memory. The caller owns every buffer,
 *   including the KV cache and the decode workspace.
 * - Kernels never trap and never wait without bound: a device-side wait that
 *   exceeds its limit records SA_ERR_TIMEOUT in a device status word and the
 *   kernel returns; read it with sa_get_device_status().
 *
 * Position / mask contract (MoE-Xtend README, "DESIGN CONTRACTS" and
 * "ATTENTION STACK"): a call that starts at cache offset `off` handles query
 * rows i = 0..T-1 at global positions p = off + i. RoPE uses p (never reset
 * per window, no wrap). Row i may attend cache row j iff j <= p and, on
 * windowed calls (window > 0), j > p - window (the band i-W<j<=i of the GQA
 * Attention study note). The layer schedule (window on even layers, full on
 * odd ones) is the caller's choice of `window`.
 */
#ifndef SINKATTN_H
#define SINKATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sa_stream_t; /* == cudaStream_t */

typedef enum sa_status {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,      /* null pointer, bad stride/alignment, T or B < 0 ... */
  SA_ERR_SHAPE = 2,            /* n_q % n_kv != 0, d not in {64, 96, 128}, q_mult > 16 */
  SA_ERR_CAPACITY = 3,         /* offset + T > cache capacity, or position >= max_pos */
  SA_ERR_OFFSET_MISMATCH = 4,  /* the call's offset differs from cache->offset */
  SA_ERR_STALE_SNAPSHOT = 5,   /* restore after rows below the snapshot were rewritten */
  SA_ERR_CUDA = 6,             /* a CUDA runtime/driver call failed (launch, tensor map) */
  SA_ERR_TIMEOUT = 7,          /* a bounded device wait ran out (read via sa_get_device_status) */
  SA_ERR_WORKSPACE = 8,        /* decode workspace missing or too small */
  SA_ERR_UNSUPPORTED = 9       /* operation not provided for this cache format (prefill on FP8) */
} sa_status;

/* Element format of a cache (sa_kv_cache.kv_dtype). */
typedef enum sa_kv_dtype {
  SA_KV_BF16 = 0,      /* bf16 rows */
  SA_KV_FP8_E4M3 = 1   /* e4m3 codes + one fp32 scale per row (sa_kv_cache_init_fp8) */
} sa_kv_dtype;

/* Capacity of the cache's overwrite log (see sa_kv_restore). */
#define SA_KV_LOG_CAP 32

/*
 * One layer's KV cache (MoE-Xtend README, "NOTATION": K,V [B, T_cache, H_kv, d];
 * "KV CACHE": preallocated, Cache.extend writes rows [offset, offset+t) then
 * advances offset; Cache.snapshot / Cache.restore).
 *
 * k, v : device, bf16, dense [B][n_kv][cap][d] (head-major), caller-owned.
 *        Row j of KV head g of sequence b is k + ((b*n_kv + g)*cap + j)*d.
 *        The pages write the cache as [B, T_cache, H_kv, d]; this library
 *        keeps each (sequence, KV head) as one contiguous run of rows so that
 *        decode streams it at full HBM bandwidth. K rows hold ROTATED keys,
 *        V rows unrotated values (GPT-OSS-Lite visual guide, "Overview":
 *        decode stores rotated K and unchanged V).
 * offset: rows [0, offset) are valid. Host-authoritative: the library updates
 *        it when an append is enqueued.
 * ring  : 0 for the linear cache above (position j in row j, offset <= cap).
 *        > 0 for a ring cache serving band layers of exactly `ring` keys
 *        (the pages' sliding-window KV reduction; MoE-Xtend README, "KV
 *        CACHE" sizing): position p lives in row p mod cap, positions are
 *        unbounded, and the cache holds the last cap positions (cap a
 *        multiple of 384, cap >= ring). Calls on a ring cache must use
 *        window == ring. Initialise with sa_kv_cache_init_ring.
 * kv_dtype, k_scale, v_scale: SA_KV_BF16 with NULL scales, or
 *        SA_KV_FP8_E4M3: k and v then hold e4m3 codes (one byte per element,
 *        same [B][n_kv][cap][d] layout) and k_scale / v_scale fp32
 *        [B][n_kv][cap] row scales (see sa_kv_cache_init_fp8).
 * The remaining fields are bookkeeping for snapshot/restore; initialise the
 * whole struct with sa_kv_cache_init (or _ring, _fp8) and do not edit them.
 */
typedef struct sa_kv_cache {
  void* k;
  void* v;
  int32_t B, cap, n_kv, d;
  int64_t offset;
  int64_t seq;          /* +1 per append and per restore */
  int64_t high_water;   /* largest offset ever reached */
  int64_t log_seq[SA_KV_LOG_CAP];  /* appends that started below high_water */
  int64_t log_row[SA_KV_LOG_CAP];
  int32_t log_len;
  int64_t log_floor_seq; /* summary of entries dropped from the full log: */
  int64_t log_floor_row; /* latest dropped seq, lowest dropped row        */
  int32_t ring;          /* 0: linear; > 0: ring cache for `ring`-key bands */
  int32_t kv_dtype;      /* sa_kv_dtype */
  void* k_scale;         /* FP8 only: fp32 [B][n_kv][cap] */
  void* v_scale;
} sa_kv_cache;

typedef struct sa_snapshot {
  uint64_t cache_id;    /* identity of the cache (its K base address) */
  int64_t offset;
  int64_t seq;
  int32_t cap;
} sa_snapshot;

/*
 * Arguments of one attention call (prefill: T >= 0 rows; decode: T == 1).
 *
 * q      : device bf16 [B][T][n_q][d] via q_strides.
 * k, v   : device bf16 [B][T][n_kv][d] via k_strides / v_strides: the call's
 *          NEW rows, appended to the cache at rows [offset, offset+T).
 * sinks  : device fp32 [n_q], one logit per query head (a raw logit compared
 *          with sm_scale*<q,k>, not itself scaled), or NULL for no sink
 *          (sink = -inf, plain softmax attention). Query head h = g*q_mult+m
 *          uses KV head g = h / q_mult and sink sinks[h].
 * offset : must equal cache->offset (the offset used for RoPE and masks).
 * window : <= 0 full causal; > 0 band of `window` keys.
 * sm_scale: score scale, e.g. 1/sqrt(d).
 * rope_fused: 1 = q and k are UNrotated and the library rotates them with
 *          cos/sin at p = offset + i; 0 = they are already rotated.
 * cos, sin: device fp32 [max_pos][d/2] tables from sa_yarn_rope_tables
 *          (concentration folded in); required when rope_fused = 1 (needs
 *          offset + T <= max_pos), ignored otherwise.
 * out    : device bf16 [B][T][n_q][d] via out_strides.
 * lse    : device fp32 [B][n_q][T] or NULL: ln(sum_j e^{s_j} + e^{sink}).
 */
typedef struct sa_attn_args {
  const void* q;   int64_t q_strides[3];
  const void* k;   int64_t k_strides[3];
  const void* v;   int64_t v_strides[3];
  const float* sinks;
  int32_t B, T, n_q;
  int64_t offset;
  int32_t window;
  float sm_scale;
  int32_t rope_fused;
  const float* cos; const float* sin; int32_t max_pos;
  void* out;       int64_t out_strides[3];
  float* lse;
} sa_attn_args;

/* Human-readable name of a status code (static string). */
const char* sa_status_string(sa_status s);

/*
 * YaRN / NTK-by-parts rotary tables (MoE-Xtend README, "ROPE + SCALING").
 * For pair i < d/2 and position t < max_pos:
 *   freq_i = theta^(i/(d/2)); extrap = 1/freq_i; interp = 1/(scaling*freq_i);
 *   i_beta  = (d/2) ln(orig_ctx/(beta*2pi)) / ln(theta);
 *   i_alpha = (d/2) ln(orig_ctx/(alpha*2pi)) / ln(theta);
 *   mask = 1 - clamp((i - i_beta)/(i_alpha - i_beta), 0, 1);
 *   inv_freq = interp*(1-mask) + extrap*mask;  conc = 0.1 ln(scaling) + 1;
 *   cos[t][i] = conc*cos(t*inv_freq), sin[t][i] = conc*sin(t*inv_freq).
 * Angles are formed in fp64 and the results rounded to fp32.
 * cos_out, sin_out: device fp32 [max_pos][d/2], caller-owned.
 * Errors: SA_ERR_INVALID_ARG (null, max_pos < 1, d odd or < 2, theta <= 1,
 * scaling <= 0, orig_ctx < 1, alpha/beta <= 0, alpha >= beta).
 */
sa_status sa_yarn_rope_tables(float* cos_out, float* sin_out, int32_t max_pos, int32_t d,
                              double theta, double scaling, int32_t orig_ctx,
                              double alpha, double beta, sa_stream_t stream);

/*
 * In-place RoPE of Q and K (MoE-Xtend README, "DESIGN CONTRACTS": positions
 * t = offset + local_t). Half-split pairs (x[c], x[c+d/2]):
 *   x1' = x1*cos - x2*sin, x2' = x2*cos + x1*sin  (fp32, rounded to bf16).
 * q: device bf16 [B][T][n_q][d] (q_strides), k: [B][T][n_kv][d] (k_strides);
 * either may be NULL to skip it. Requires offset + T <= max_pos.
 */
sa_status sa_rope_apply_qk(void* q, const int64_t q_strides[3], void* k, const int64_t k_strides[3],
                           int32_t B, int32_t T, int32_t n_q, int32_t n_kv, int32_t d, int64_t offset,
                           const float* cos, const float* sin, int32_t max_pos, sa_stream_t stream);

/* Initialise a cache descriptor over caller-owned K/V buffers (offset 0). */
sa_status sa_kv_cache_init(sa_kv_cache* cache, void* k, void* v, int32_t B, int32_t cap,
                           int32_t n_kv, int32_t d);

/*
 * Ring cache for band layers of `window` keys (see `ring` above): k, v as
 * for sa_kv_cache_init with cap rows per (sequence, KV head), cap a multiple
 * of 384 and >= window (SA_ERR_SHAPE otherwise). The buffers must be zeroed
 * before first use (rows never written are read, masked, by the kernels).
 * Appends of T rows need T <= cap; a prefill of T rows needs
 * T + window - 1 <= cap (the keys of the call's first row must survive the
 * call's own appends); otherwise SA_ERR_CAPACITY. A snapshot can be restored
 * while the rows its band needs, positions [offset - window + 1, offset),
 * have not been overwritten (else SA_ERR_STALE_SNAPSHOT).
 */
sa_status sa_kv_cache_init_ring(sa_kv_cache* cache, void* k, void* v, int32_t B, int32_t cap,
                                int32_t n_kv, int32_t d, int32_t window);

/*
 * FP8 cache: quantised K/V rows with the dequantisation fused into decode
 * (MoE-Xtend README, "ROADMAP": quantisation-aware long-context runs,
 * bandwidth first -- KV plus its dequantisation). Decode reads 1 byte per
 * element plus 8 bytes of scales per (position, KV head) instead of 2 bytes.
 * k, v    : device e4m3 codes [B][n_kv][cap][d], 16-byte aligned.
 * k_scale, v_scale: device fp32 [B][n_kv][cap], 16-byte aligned.
 * window  : 0 for a linear cache, > 0 for a ring cache of `window`-key
 *           bands (same rules as sa_kv_cache_init_ring).
 * cap must be a multiple of 16 (SA_ERR_SHAPE). Every stored row x (K after
 * rotation, V as given, each the bf16 row a bf16 cache would hold) is kept
 * as scale = fl32(amax|x| / 448) and codes e4m3(fl32(x_d / scale)) rounded
 * to nearest even with saturation (a zero row: scale 0, codes 0); readers
 * see code * scale. Appends (sa_kv_append, and the new row of
 * sa_attn_decode, which also attends its quantised value) quantise;
 * sa_attn_prefill returns SA_ERR_UNSUPPORTED on an FP8 cache: run prefill
 * on a bf16 cache and move its rows over with sa_kv_append (strides
 * {n_kv*cap*d, d, cap*d} describe a bf16 cache as [B][T][n_kv][d]).
 * Buffers of a ring cache, scales included, must be zeroed before first use.
 */
sa_status sa_kv_cache_init_fp8(sa_kv_cache* cache, void* k, void* v, void* k_scale, void* v_scale,
                               int32_t B, int32_t cap, int32_t n_kv, int32_t d, int32_t window);

/*
 * Append T already-rotated K rows and V rows at [offset, offset+T), then
 * offset += T (MoE-Xtend README, "KV CACHE": Cache.extend). k_rot/v: device
 * bf16 [B][T][n_kv][d] via strides. Bit copy into a bf16 cache; into an FP8
 * cache each row is quantised (sa_kv_cache_init_fp8). SA_ERR_CAPACITY if
 * offset + T > cap.
 */
sa_status sa_kv_append(sa_kv_cache* cache, const void* k_rot, const int64_t k_strides[3],
                       const void* v, const int64_t v_strides[3], int32_t T, sa_stream_t stream);

/* Capture the cache state (offset; rows below it are immutable under
 * append-only use). Host only, no device work. */
sa_status sa_kv_snapshot(const sa_kv_cache* cache, sa_snapshot* out);

/*
 * Reinstate a snapshot ("prefill once, decode many"): rolls the offset back
 * to snap->offset. Host only. SA_ERR_STALE_SNAPSHOT when some row below
 * snap->offset was rewritten after the snapshot (a restore to a lower
 * offset followed by an append). The log keeps the last SA_KV_LOG_CAP such
 * rewrites exactly and summarises older ones conservatively (a snapshot
 * older than a dropped rewrite, with rows above that rewrite's first row, is
 * reported stale). SA_ERR_INVALID_ARG for another cache's snapshot.
 */
sa_status sa_kv_restore(sa_kv_cache* cache, const sa_snapshot* snap);

/*
 * Prefill: rotate (if rope_fused) and append the call's K/V rows to the
 * cache, then attend the T query rows to cache rows [0, offset+T) with the
 * per-head sink column (MoE-Xtend README, "ATTENTION STACK": softmax over
 * [QK + B, S], sink column dropped after normalisation; GQA Attention study
 * note, "How it works"). cache->offset += T on success. T == 0 is a no-op.
 * The attention runs on tcgen05 tensor cores with fp32 accumulation; the
 * softmax weights enter the PV product as bf16.
 * When rope_fused, one launch rotates the K rows as it appends them and
 * stages the rotated queries in args->out (same [B][T][n_q][d] view); the
 * attention kernel then loads its query tiles from there and overwrites each
 * staged tile with its own output rows, so `out` may be `q` itself but must
 * not overlap k, v, the cache, the sinks, the tables or lse otherwise. Two
 * launches on `stream` (staging, attention). The
 * attention kernel schedules its work items from a device
 * counter. The library keeps 128 such counters per device and never lets two
 * calls in flight share one: calls made outside stream capture take the
 * first 64 round robin, and before one reuses a counter its stream waits for
 * the event the library recorded after that counter's previous call (on
 * whatever stream it ran). Calls captured into a CUDA graph take the other
 * 64 round robin without events; graph replays that run at the same time as
 * one another must hold at most 64 prefill calls between them.
 * Band layers of d = 64 whose window is narrow enough for the query heads of
 * a KV group to share one key window of at most 160 columns (128/q_mult +
 * window + 14 <= 160: W up to 130, 114, 82 or 18 for q_mult 8, 4, 2 or 1)
 * take a second kernel instead: the staging launch only
 * appends K/V, the kernel reads q directly and rotates it itself, no
 * schedule counter is used, and `out` may again be `q` itself.
 * SA_ERR_UNSUPPORTED on an FP8 cache.
 */
sa_status sa_attn_prefill(sa_kv_cache* cache, const sa_attn_args* args, sa_stream_t stream);

/*
 * Decode: one new row per sequence (args->T must be 1). Rotates q and k,
 * appends the new K/V row at cache row `offset`, and attends to cache rows
 * [max(0, offset+1-window), offset] (all rows when window <= 0), split
 * across SMs. cache->offset += 1 on success (MoE-Xtend README, "DESIGN
 * CONTRACTS": exactly one row per layer per step). On an FP8 cache the
 * kernel dequantises K/V as it reads them and stores and attends the new
 * row quantised; queries enter the QK product as f16 after an exact
 * per-head power-of-two scaling, and the scaled softmax weights enter the PV
 * product as f16.
 * The rows are shared out among the CTAs of each (sequence, KV head) at run
 * time (the CTAs that stream faster take more), so the fp32 partial sums are
 * grouped differently from call to call: two identical calls can differ in
 * the last bit of an output, each within the same rounding of the exact
 * value.
 * workspace: device memory of at least sa_attn_decode_workspace_size()
 *   bytes, caller-owned, ZERO-FILLED before its first use; the kernel leaves
 *   it zeroed again on completion. Calls that share a workspace must not
 *   overlap on the device (order them on one stream).
 */
sa_status sa_attn_decode(sa_kv_cache* cache, const sa_attn_args* args, void* workspace,
                         size_t workspace_bytes, sa_stream_t stream);

/* Workspace bytes sa_attn_decode needs for B sequences of n_q/n_kv heads of
 * width d on any device with at most 256 SMs. */
size_t sa_attn_decode_workspace_size(int32_t B, int32_t n_q, int32_t n_kv, int32_t d);

/*
 * Decode for callers that cannot allocate device memory: an embedded runtime
 * without its own allocator, code that must not call cudaMalloc in its
 * serving loop, or a host process that only ever receives device pointers
 * from someone else. The pages have no counterpart to this entry point.
 *
 * Same operation, arguments and results as sa_attn_decode, but the split
 * scratch lives in a fixed array inside the library (a file-scope
 * __device__ array of SA_DECODE_STATIC_SCRATCH_BYTES bytes, which every GPU
 * that loads the library holds until the process exits). No call allocates:
 * no cudaMalloc, cudaFree or allocating library routine.
 * - The first call on a device (with that device current) looks up the
 *   array's device address and zeroes it once; make that first call before
 *   any stream capture.
 * - SA_ERR_WORKSPACE when this call's split scratch would exceed
 *   SA_DECODE_STATIC_SCRATCH_BYTES (large B * n_kv * q_mult * d); use
 *   sa_attn_decode with a workspace then.
 * - Every call shares the one array: calls that overlap on the GPU (other
 *   streams, other threads) race. Order them on one stream.
 */
#define SA_DECODE_STATIC_SCRATCH_BYTES (1u << 20)
sa_status sa_attn_decode_static(sa_kv_cache* cache, const sa_attn_args* args, sa_stream_t stream);

/*
 * Backward pass of sink-augmented GQA attention, for a sequence attending to
 * itself (a training step: no cache prefix, positions 0..T-1), on the
 * ROTATED q and k the forward used (GPT-OSS-Lite README, "Architecture":
 * learned attention sinks, trained end to end). With P the forward's softmax
 * weights (sink column included in the normalisation), D_i = <dO_i, o_i>
 * and dS = P (dO V^T - D):
 *   dq = sm_scale dS K,  dk = sm_scale dS^T Q,  dv = P^T dO
 *   (dk, dv summed over the q_mult heads of each KV group),
 *   dsinks[h] = -sum_{b,i} exp(sinks[h] - lse[b][h][i]) D_i.
 * Gradients with respect to unrotated q, k: apply sa_rope_apply_qk with the
 * sin table negated (the rotation's transpose).
 *
 * q, k, v, out (the forward's output), d_out: device bf16 [B][T][H][d] via
 *   strides (inner dimension contiguous, strides multiples of 8), 16-byte
 *   aligned.
 * lse    : the forward's fp32 [B][n_q][T] log-sum-exp (sa_attn_prefill's lse).
 * sinks  : fp32 [n_q] or NULL (no sink; dsinks is then not written).
 * window : <= 0 full causal, > 0 band of `window` keys.
 * dq     : fp32 [B][T][n_q][d] dense; dk, dv: fp32 [B][T][n_kv][d] dense;
 *   dsinks: fp32 [n_q] (overwritten) or NULL. All outputs are written, not
 *   accumulated into.
 * workspace: device memory of sa_attn_backward_workspace_size() bytes
 *   (16-byte aligned, contents irrelevant).
 * Products run on the tensor cores (bf16 operands, fp32 accumulation); P and
 * dS enter their products as bf16. dq (summed over 128-key tiles by
 * reduce-adds) and dsinks (summed over blocks by atomics) add in a varying
 * order, so they can differ in the last bits between calls; dk and dv do
 * not. Errors: SA_ERR_INVALID_ARG (null,
 * misaligned, bad stride, B/T/n_q < 1), SA_ERR_SHAPE (d not in {64, 96,
 * 128}, n_q % n_kv != 0, n_q > 8192, ceil(T / 128) n_kv B >= 2^31),
 * SA_ERR_WORKSPACE (too small), SA_ERR_CUDA.
 */
typedef struct sa_attn_bwd_args {
  const void* q;     int64_t q_strides[3];
  const void* k;     int64_t k_strides[3];
  const void* v;     int64_t v_strides[3];
  const void* out;   int64_t out_strides[3];
  const void* d_out; int64_t d_out_strides[3];
  const float* lse;
  const float* sinks;
  int32_t B, T, n_q, n_kv, d;
  int32_t window;
  float sm_scale;
  float* dq;
  float* dk;
  float* dv;
  float* dsinks;
} sa_attn_bwd_args;

sa_status sa_attn_backward(const sa_attn_bwd_args* args, void* workspace, size_t workspace_bytes,
                           sa_stream_t stream);
size_t sa_attn_backward_workspace_size(int32_t B, int32_t T, int32_t n_q);

/*
 * The dense projections around the attention (GQA Attention study note, "How
 * it works": the residual stream x [T, 2880] goes through pre-norm RMSNorm
 * and one fused linear qkv of width d_h (n_q + 2 n_kv) = 5120 whose columns
 * are q, then k, then v; after attention the heads, flattened to [T, 4096],
 * go through the linear out back to [T, 2880], added to the residual; both
 * linears are bf16 with bias). Matrices are row-major bf16 with leading
 * dimensions (ld*, in elements, multiples of 8, >= the row width); bases
 * 16-byte aligned. Weights follow nn.Linear: W [N][K], y = x W^T + b. The
 * product runs on tcgen05 tensor cores with fp32 accumulation, one rounding
 * to bf16 at the end. Errors: SA_ERR_INVALID_ARG for a null or misaligned
 * pointer, a bad leading dimension, M < 0, N or K < 1; SA_ERR_CUDA if a
 * launch fails. M == 0 is a no-op.
 */

/*
 * Fold RMSNorm's gain into the qkv weight, once per model: w_folded[n][k] =
 * bf16(w[n][k] * gamma[k]) (the product formed exactly, rounded once).
 * w, w_folded: [N][K] bf16 (ld ldw / ldf); gamma: fp32 [K]. May be in place.
 */
sa_status sa_rmsnorm_fold_weight(const void* w, int64_t ldw, const float* gamma, void* w_folded,
                                 int64_t ldf, int32_t N, int32_t K, sa_stream_t stream);

/*
 * Pre-norm RMSNorm + fused qkv projection:
 *   y[m][n] = (sum_k x[m][k] w_folded[n][k]) / sqrt(mean_k x[m][k]^2 + eps) + bias[n]
 * which is RMSNorm(x; gamma, eps) W^T + b with w_folded from
 * sa_rmsnorm_fold_weight. x [M][K], y [M][N] (e.g. the fused q|k|v rows
 * that sa_attn_prefill / sa_attn_decode take as strided views), bias bf16
 * [N] or NULL, eps >= 0. The row statistics come from the same x tiles the
 * product reads; the normalised x is never written. y must not overlap x.
 */
sa_status sa_qkv_proj(const void* x, int64_t ldx, const void* w_folded, int64_t ldw, const void* bias,
                      float eps, void* y, int64_t ldy, int32_t M, int32_t N, int32_t K, sa_stream_t stream);

/*
 * Out projection with the residual add, in place: x[m][n] += sum_k
 * o[m][k] w[n][k] + bias[n] (the sum, the bias and the old x added in fp32,
 * rounded once). o [M][K] (the attention output flattened over heads),
 * w [N][K], bias bf16 [N] or NULL, x [M][N] the residual stream. o must not
 * overlap x.
 */
sa_status sa_out_proj(const void* o, int64_t ldo, const void* w, int64_t ldw, const void* bias, void* x,
                      int64_t ldx, int32_t M, int32_t N, int32_t K, sa_stream_t stream);

/*
 * Reads and clears the device status word of the current device (waits for
 * the device to be idle). *code receives SA_OK or SA_ERR_TIMEOUT.
 */
sa_status sa_get_device_status(int32_t* code);

/*
 * Upper bound, in SM clock cycles, of every device-side wait of later
 * launches on the current device (default about one second). For tests of
 * the timeout path only.
 */
sa_status sa_set_wait_limit(int64_t cycles);

/*
 * Which of the 128 schedule counters (sa_attn_prefill above) the index-th
 * prefill call on a device takes: index counts the calls made outside
 * stream capture (captured == 0) or inside it (captured != 0) separately.
 * Pure host arithmetic, no device work (no counterpart in the method;
 * exposes the allocation rule to tests).
 */
int32_t sa_prefill_sched_slot(uint64_t index, int32_t captured);

/*
 * Timing hook for the attention kernel of sa_attn_prefill (no counterpart in
 * the method; measurement support). While set, every sa_attn_prefill call
 * records `before` on its stream after the staging launch (RoPE + append)
 * and just before the attention kernel, and `after` just after it, so the
 * caller can time the attention kernel alone with cudaEventElapsedTime.
 * before/after: cudaEvent_t handles owned by the caller, both NULL to clear
 * (one NULL and one not: SA_ERR_INVALID_ARG). Process-wide; not for
 * concurrent use from several threads.
 */
sa_status sa_set_prefill_events(void* before, void* after);

#ifdef __cplusplus
}
#endif

#endif /* SINKATTN_H */
