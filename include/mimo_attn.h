/*
 * mimo_attn.h -- C ABI of the MiMo-V2-Flash hybrid attention operator for
 * NVIDIA B200 (sm_100a).
 *
 * What the operator computes (MiMo-V2-Flash model doc, "Key features":
 * hybrid attention bullet; MiMoV2FlashConfig parameters num_attention_heads,
 * num_key_value_heads, head_dim, v_head_dim, sliding_window):
 *
 *   causal grouped-query attention, Hq query heads over Hkv key/value heads
 *   (query head h reads key/value head h / (Hq/Hkv)), query/key dim Dqk and
 *   value dim Dv, softmax scale s (default 1/sqrt(Dqk)), an optional sliding
 *   window, and a per-query-head attention-sink logit sigma_h:
 *
 *     visible(i, j)  <=>  0 <= i - j  and  (window == 0 or i - j <= window-1)
 *     S_j  = s * <q_i, k_j>                         over visible j
 *     m    = max(sigma_h, max_j S_j)
 *     Z    = exp(sigma_h - m) + sum_j exp(S_j - m)
 *     out  = v_scale * sum_j exp(S_j - m) v_j / Z   (the sink has no value)
 *     lse  = m + ln Z                                (natural log, with sink)
 *
 *   window = 129 is the model's sliding-window layer (the query plus the
 *   previous 128 keys); window = 0 is its global layer.  Layers interleave
 *   5 sliding-window : 1 global; the caller passes the layer's window.
 *   The sink formula is this library's reading: the documentation names a
 *   "learnable attention sink bias" but prints no formula.
 *
 * Conventions for every entry point
 *   - Supported shapes: Dqk == 192, Dv == 128, Hq % Hkv == 0, Hq/Hkv <= 16
 *     for decode; other shapes return MIMO_ERR_UNSUPPORTED.
 *   - All tensor arguments are caller-owned DEVICE pointers, contiguous,
 *     16-byte aligned.  The library keeps no pointer after the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  No host synchronisation happens.
 *     The return status covers argument validation and launch errors;
 *     a fault inside a kernel surfaces at the caller's next synchronisation.
 *   - Every wait inside a kernel is bounded.  A wait that gives up records
 *     MIMO_ERR_TIMEOUT in a device status word, which
 *     mimo_attn_device_status() reads and clears.
 *   - On a non-OK status, mimo_attn_last_error() returns a message for the
 *     calling thread.
 */
#ifndef MIMO_ATTN_H_
#define MIMO_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MIMO_OK = 0,
  MIMO_ERR_INVALID_ARG = 1,   /* NULL pointer, negative size, bad window ... */
  MIMO_ERR_UNSUPPORTED = 2,   /* head dims other than 192/128, group > 16 ... */
  MIMO_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  MIMO_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than required */
  MIMO_ERR_TIMEOUT = 5,       /* a bounded in-kernel wait gave up */
  MIMO_ERR_BOUNDS = 6         /* checked build only: an index outside its buffer (access skipped) */
} mimo_status_t;

typedef enum { MIMO_DTYPE_BF16 = 0, MIMO_DTYPE_F32 = 1 } mimo_dtype_t;

typedef struct {
  int num_heads_q;     /* Hq  (64 in the model) */
  int num_heads_kv;    /* Hkv (4 in the model)  */
  int head_dim_qk;     /* Dqk (192) */
  int head_dim_v;      /* Dv  (128) */
  float softmax_scale; /* <= 0 selects 1/sqrt(Dqk) */
  float v_scale;       /* output multiplier (attention_value_scale); 0 selects 1 */
  int out_dtype;       /* mimo_dtype_t of `out` */
} mimo_attn_dims_t;

/*
 * Packed variable-length prefill (one attention layer over all prompt tokens).
 *
 *   q          [total_tokens, Hq,  Dqk] bf16, post-RoPE
 *   k          [total_tokens, Hkv, Dqk] bf16, post-RoPE
 *   v          [total_tokens, Hkv, Dv ] bf16
 *   sinks      [Hq] fp32 sink logits (natural-log units), or NULL for none
 *   window     0 = global causal; >= 1 = the query plus window-1 earlier keys
 *   cu_seqlens [num_seqs + 1] int32 on the device: cu[0] = 0, non-decreasing,
 *              cu[num_seqs] = total_tokens.  Sequence s owns tokens
 *              [cu[s], cu[s+1]); lengths of 0 are allowed.
 *   max_seqlen >= every sequence length (sizes the launch; not read back)
 *   out        [total_tokens, Hq, Dv] in dims->out_dtype
 *   lse        [Hq, total_tokens] fp32, or NULL to skip
 *
 * Work is split over (sequence, 128-query tile, pair of query heads of one
 * key/value group).  Key tiles wholly outside the window are never loaded.
 */
mimo_status_t mimo_attn_prefill(const mimo_attn_dims_t* dims,
                                const void* q, const void* k, const void* v,
                                const float* sinks, int window,
                                const int32_t* cu_seqlens, int num_seqs,
                                int total_tokens, int max_seqlen,
                                void* out, float* lse, void* stream);

/*
 * Bytes of device workspace mimo_attn_decode needs for these sizes
 * (split-KV partial results).  0 when one split covers every sequence.
 *
 * The split plan depends only on these sizes and the current device's SM
 * count (148 on B200, also assumed when no device is visible): about two
 * work units per SM, splits of 256..16384 keys, one split for a ring cache.
 * For tuning, the environment variable MIMO_DECODE_CHUNK (keys per split,
 * rounded up to a multiple of 64; read once per process) overrides the split
 * size; this size query and the decode call then follow the same plan.
 */
size_t mimo_attn_decode_workspace_size(const mimo_attn_dims_t* dims, int batch,
                                       int capacity, int window);

/*
 * One decode step: one query token per sequence against its KV cache
 * (MiMoV2FlashModel.forward, past_key_values: only the new token is fed).
 *
 *   q          [batch, Hq, Dqk] bf16, post-RoPE
 *   k_cache    [batch, capacity, Hkv, Dqk] bf16
 *   v_cache    [batch, capacity, Hkv, Dv ] bf16
 *   seqlens    [batch] int32 on the device: tokens so far INCLUDING the
 *              current one, whose K/V are already in the cache; the query
 *              sits at position L-1.
 *   window     0 = global.  If window > 0 and capacity == window the cache is
 *              a RING: token p lives in slot p mod capacity and every slot
 *              below min(L, capacity) is visible.  Otherwise the cache is
 *              LINEAR (slot = position) and requires L <= capacity; slots
 *              [max(0, L-window), L) are visible (all of [0, L) if window=0).
 *              L > capacity on a linear cache is clamped to capacity and
 *              recorded as MIMO_ERR_INVALID_ARG in the device status word.
 *   sinks      [Hq] fp32 or NULL
 *   out        [batch, Hq, Dv] in dims->out_dtype
 *   lse        [batch, Hq] fp32 or NULL
 *   workspace  device scratch of at least mimo_attn_decode_workspace_size()
 *              bytes (may be NULL when that size is 0).  Calls sharing one
 *              workspace must not overlap on the GPU.
 *
 * Slots past a sequence's length are never read into the result (their
 * contents may be anything, NaN included).
 */
mimo_status_t mimo_attn_decode(const mimo_attn_dims_t* dims, const void* q,
                               const void* k_cache, const void* v_cache,
                               const int32_t* seqlens, int batch, int capacity,
                               int window, const float* sinks, void* out,
                               float* lse, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * The decode step's rotation and cache write for the new token (run before
 * mimo_attn_decode on the same stream).  MiMoV2FlashConfig.rope_parameters
 * (rope_theta) and MiMoV2FlashModel.forward (position_ids, past_key_values);
 * the pages fix neither theta nor the pairing, and this library takes
 * RoFormer's rotation in the rotate-half arrangement: for i < rotary_dim/2,
 * dimensions i and i + rotary_dim/2 turn by p * theta^(-2 i / rotary_dim) at
 * the token's position p = seqlens[b] - 1; dimensions >= rotary_dim are left
 * unchanged.
 *
 *   q          [batch, Hq, Dqk] bf16: the new token's queries, rotated IN PLACE
 *   k_new      [batch, Hkv, Dqk] bf16: its keys before rotation
 *   v_new      [batch, Hkv, Dv ] bf16: its values
 *   k_cache    [batch, capacity, Hkv, Dqk] bf16: the rotated key is written
 *              to slot p (linear) or p mod capacity (ring: window > 0 and
 *              capacity == window); no other slot is touched
 *   v_cache    [batch, capacity, Hkv, Dv ] bf16: the value, same slot
 *   seqlens    [batch] int32 on the device: tokens INCLUDING the new one
 *   rope_theta > 0; rotary_dim even, 0..Dqk (0 = no rotation, plain append)
 *
 * Angles are formed in double precision.  A sequence with seqlens < 1, or
 * with p >= capacity on a linear cache, is skipped and recorded as
 * MIMO_ERR_INVALID_ARG in the device status word.
 */
mimo_status_t mimo_attn_rope_append(const mimo_attn_dims_t* dims, void* q,
                                    const void* k_new, const void* v_new,
                                    void* k_cache, void* v_cache,
                                    const int32_t* seqlens, int batch, int capacity,
                                    int window, float rope_theta, int rotary_dim,
                                    void* stream);

/*
 * Merge of decode results over disjoint parts of each sequence's keys
 * (context parallelism: a global layer's cache split across GPUs, each part
 * decoded with mimo_attn_decode, window 0, sinks = NULL, fp32 out and lse,
 * then gathered).  MiMo-V2-Flash model doc, "Key features" (learnable sink):
 *
 *   M   = max(sigma_h, max_r lse_r)
 *   Z   = exp(sigma_h - M) + sum_r exp(lse_r - M)
 *   out = dims->v_scale * sum_r exp(lse_r - M) out_r / Z,   lse = M + ln Z
 *
 *   part_out [num_parts, batch, Hq, Dv] fp32 (16-byte aligned)
 *   part_lse [num_parts, batch, Hq] fp32, natural log; -inf marks a part
 *            with no keys for that sequence (its part_out is then ignored)
 *   sinks    [Hq] fp32 or NULL;  out [batch, Hq, Dv] in dims->out_dtype;
 *   lse      [batch, Hq] fp32 or NULL
 *
 * The parts' order does not matter.  With every part empty and no sink the
 * output is 0 and lse -inf.
 */
mimo_status_t mimo_attn_decode_merge(const mimo_attn_dims_t* dims, const float* part_out,
                                     const float* part_lse, int num_parts, int batch,
                                     const float* sinks, void* out, float* lse,
                                     void* stream);

/*
 * Workspace bytes for mimo_attn_prefill_backward: 2 * Hq * total_tokens fp32.
 */
size_t mimo_attn_prefill_backward_workspace_size(const mimo_attn_dims_t* dims,
                                                 int total_tokens);

/*
 * Gradients of mimo_attn_prefill (training).  MiMo-V2-Flash model doc, "Key
 * features": the attention-sink bias is learnable, so it has a gradient.
 * Per query head h, row i, visible key j (S = s <q_i, k_j>, P = exp(S - lse_i)):
 *   D_i = <dO_i, O_i>;  dS_ij = P_ij (v_scale <dO_i, v_j> - D_i)
 *   dq_i = s sum_j dS_ij k_j;  dk_j = s sum dS_ij q_i;  dv_j = v_scale sum P_ij dO_i
 *   (dk, dv summed over the query heads of j's key/value head)
 *   dsinks_h = -sum_i exp(sinks_h - lse_i) D_i
 *
 *   q, k, v, sinks, window, cu_seqlens, num_seqs, total_tokens, max_seqlen:
 *              as passed to mimo_attn_prefill
 *   out, lse   the forward's out (dims->out_dtype) and lse [Hq, total_tokens]
 *   dout       [total_tokens, Hq, Dv], same dtype as out
 *   dq         [total_tokens, Hq,  Dqk] fp32;  dk [total_tokens, Hkv, Dqk] fp32
 *   dv         [total_tokens, Hkv, Dv ] fp32 (all three overwritten)
 *   dsinks     [Hq] fp32, required when sinks is given (ignored otherwise)
 *   workspace  >= mimo_attn_prefill_backward_workspace_size() bytes, 16-byte aligned
 *
 * Tensor-core kernels with bf16 operands and fp32 accumulation (dK and dV
 * on tcgen05 when out / dout are bf16, warp-level mma.sync otherwise and for
 * dq); P, dS and dO are rounded to bf16 as operands (fp32 dO included) and D
 * is computed from that rounded dO; deterministic: no atomics, fixed
 * summation order.
 *
 * All buffers are caller-owned device memory; the call is asynchronous on
 * `stream`.  Errors, returned before any launch: the dims rules of
 * mimo_attn_prefill (MIMO_ERR_UNSUPPORTED / MIMO_ERR_INVALID_ARG); window < 0,
 * negative sizes, cu_seqlens NULL, any of q, k, v, out, lse, dout, dq, dk, dv
 * NULL, dsinks NULL while sinks is given, tensors not 16-byte aligned (lse,
 * sinks, dsinks 4-byte), or max_seqlen > total_tokens -> MIMO_ERR_INVALID_ARG;
 * num_seqs > 65535 -> MIMO_ERR_UNSUPPORTED; a missing or small workspace ->
 * MIMO_ERR_WORKSPACE.  total_tokens, num_seqs or max_seqlen of 0 is a no-op
 * returning MIMO_OK.  max_seqlen must be at least the longest sequence.
 */
mimo_status_t mimo_attn_prefill_backward(const mimo_attn_dims_t* dims, const void* q,
                                         const void* k, const void* v, const void* out,
                                         const float* lse, const void* dout,
                                         const float* sinks, int window,
                                         const int32_t* cu_seqlens, int num_seqs,
                                         int total_tokens, int max_seqlen, float* dq,
                                         float* dk, float* dv, float* dsinks,
                                         void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * Workspace bytes for mimo_attn_decode_fp8 (the same split plan as the bf16
 * decode, so the same size).
 */
size_t mimo_attn_decode_fp8_workspace_size(const mimo_attn_dims_t* dims,
                                           int batch, int capacity, int window);

/*
 * One decode step against an FP8 KV cache (MiMo-V2-Flash model doc, "Key
 * features": FP8 mixed precision; the cache format is this library's own).
 *
 *   k_cache    [batch, capacity, Hkv, Dqk] e4m3 bytes (OCP FP8 E4M3: sign,
 *              4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 *              S.1111.111 = NaN, largest finite 448)
 *   v_cache    [batch, capacity, Hkv, Dv ] e4m3 bytes
 *   k_scale    [Hkv] fp32 on the device: key element = code * k_scale[g]
 *   v_scale_kv [Hkv] fp32 on the device: value element = code * v_scale_kv[g]
 *              (g = the key/value head; one pair of scales per layer and head)
 *
 * Every other argument, the ring/linear cache rules, the workspace and the
 * error behaviour are those of mimo_attn_decode.  The products run in f16
 * with fp32 accumulation: e4m3 codes convert to f16 exactly, q is rounded to
 * f16 once (q elements must lie within the f16 range, |q| < 65504), and the
 * softmax weights are rounded to f16 for the P.V product.  k_scale and
 * v_scale_kv must be non-NULL and 4-byte aligned (else MIMO_ERR_INVALID_ARG).
 */
mimo_status_t mimo_attn_decode_fp8(const mimo_attn_dims_t* dims, const void* q,
                                   const void* k_cache, const void* v_cache,
                                   const float* k_scale, const float* v_scale_kv,
                                   const int32_t* seqlens, int batch, int capacity,
                                   int window, const float* sinks, void* out,
                                   float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * mimo_attn_decode without a workspace and without allocating.  The model
 * documentation has no counterpart to this call: it exists for callers that
 * cannot call cudaMalloc -- code running in a process whose device memory is
 * owned by another allocator (a serving runtime or a framework memory pool),
 * or latency-critical loops that cannot take the device synchronisation an
 * allocation may cause.  It allocates nothing and calls no allocating routine.
 *
 * Arguments are those of mimo_attn_decode minus the workspace.  The split-KV
 * partials go to a 16 MiB array compiled into the library (every GPU that
 * loads the library holds it until exit).  Sizes whose workspace
 * (mimo_attn_decode_workspace_size) exceeds 16 MiB are rejected with
 * MIMO_ERR_WORKSPACE before any device work.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  The cached address belongs to the device's context as it was at
 * that first call: after cudaDeviceReset (or anything else that destroys the
 * device's primary context) do not call this entry point again on that device
 * in the same process.  All calls share the one array and it keeps the previous call's
 * contents (nothing in it needs to start at zero): calls that overlap on the
 * GPU, on any streams, race and corrupt each other's results.
 */
mimo_status_t mimo_attn_decode_noalloc(const mimo_attn_dims_t* dims, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* seqlens, int batch, int capacity,
                                       int window, const float* sinks, void* out,
                                       float* lse, void* stream);

/* Message for the calling thread's last non-OK status ("" if none). */
const char* mimo_attn_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the device status word that
 * bounded in-kernel waits and device-side argument checks write.  Returns
 * MIMO_OK, MIMO_ERR_TIMEOUT, MIMO_ERR_INVALID_ARG, MIMO_ERR_BOUNDS (checked
 * build) or MIMO_ERR_CUDA.
 */
mimo_status_t mimo_attn_device_status(void* stream);

/*
 * Writes `code` (a mimo_status_t value) into the device status word,
 * ordered on `stream`: kernels launched on it afterwards see the new value.
 * A diagnostic hook for testing the failure path without a failing GPU.
 * With MIMO_ERR_TIMEOUT pre-loaded, every kernel that has bounded waits
 * (prefill, decode, FP8 decode, the decode combine, the tcgen05 backward)
 * returns at entry, as it does after a real timed-out wait elsewhere, and
 * writes none of its outputs.  mimo_attn_device_status() then reports the
 * code and clears it.  Codes outside 0..5 return MIMO_ERR_INVALID_ARG.
 */
mimo_status_t mimo_attn_set_device_status(int code, void* stream);

/*
 * Failure-path test hook: launches one CTA in which a thread waits on a
 * barrier that nothing arrives at.  The wait gives up after its bound (1 s),
 * records MIMO_ERR_TIMEOUT in the device status word and raises the CTA's
 * abort flag, and the CTA's teardown waits for the bulk copy another thread
 * had in flight, as the library's kernels do after a timed-out wait.  Nothing
 * faults and nothing waits without a bound.  Asynchronous on `stream`;
 * mimo_attn_device_status() then reports MIMO_ERR_TIMEOUT (and clears it).
 */
mimo_status_t mimo_attn_wait_selftest(void* stream);

/*
 * Bounds-checked build.  The same sources compiled with -DMIMO_CHECKED give
 * libmimo_attn_checked.so: every kernel checks each row index it forms for a
 * global read or write against the row count of that buffer before the
 * access.  A miss skips the access and records MIMO_ERR_BOUNDS in the device
 * status word and its site (file number * 10000 + source line) for
 * mimo_attn_checked_site().  The checks only catch indexing mistakes of the
 * library itself: the host and device argument checks above come first.  In
 * the normal build the checks compile away.
 *
 * mimo_attn_is_checked_build: 1 in the checked build, 0 otherwise.
 * mimo_attn_checked_site: synchronises `stream`, returns the first recorded
 *   site (0 if none) and clears it; always 0 in the normal build; -1 if a
 *   CUDA call failed (mimo_attn_last_error() says which).
 * mimo_attn_checked_selftest: checked build only (else MIMO_ERR_UNSUPPORTED):
 *   launches one thread that checks row 4 of a 4-row buffer and touches no
 *   memory, so that the status word then holds MIMO_ERR_BOUNDS and the site
 *   is set; asynchronous on `stream`.
 */
int mimo_attn_is_checked_build(void);
int mimo_attn_checked_site(void* stream);
mimo_status_t mimo_attn_checked_selftest(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MIMO_ATTN_H_ */
