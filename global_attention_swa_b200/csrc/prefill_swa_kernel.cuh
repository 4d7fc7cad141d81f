// Sliding-window prefill with the whole key/value group packed into the MMA
// rows (tcgen05).
//
// MiMo-V2-Flash model doc, "Key features" (sliding-window layers with a small
// window, learnable attention sink) and MiMoV2FlashConfig (64 query heads
// over 4 key/value heads, head_dim 192 / v_head_dim 128, sliding_window 129).
//
// A block is QB = 128 / G consecutive queries of one sequence times the G
// query heads of one key/value head g: 128 rows, row = query * G + head (the
// [token][head][dim] layout makes these rows one TMA box).  All G heads read
// the same keys, so one score tile covers the block.  Blocks go in pairs (2 QB
// queries): both blocks of a pair share one key window, the
// N = roundup16(W + 2 QB - 1) keys [q0 + 2 QB - N, q0 + 2 QB), loaded once,
// of which each row sees at most W (~90 % useful at W = 129, QB = 8, N = 144).
// With the whole window in one tile there is no online rescaling: max,
// exponentials and the sink's share are exact for the row.
//
//   warp 12     TMA producer: Q double-buffered (2 x 48 KB, from DRAM, one
//               block ahead), K (N x 384 B) and V (N x 256 B) once per pair.
//   warp 13     MMA issuer: S(n) = Q K^T into TMEM score buffer n & 1, then
//               O = P(n-1) V for the previous block (software pipelined).
//   warps 0-7   softmax: two warpgroups, warpgroup s takes the blocks with
//               n & 1 == s (its own score buffer), one row per thread, two
//               passes over the TMEM row (max, then exponentials), P written
//               back as bf16.  Chunks of 16 columns wholly inside the row's
//               window skip the per-element mask.
//   warps 8-11  epilogue: O / l -> bf16/fp32 rows, lse.
//
// The output is normalised by the sum of the bf16-rounded P that P.V
// multiplies (plus the sink's term).  The value operand of P.V carries a third
// 64-column block that holds ones, and the product runs with N = 144: O's
// columns 128..143 then accumulate exactly that row sum, at no extra MMA
// instruction, and the softmax warps keep only the unrounded sum (for lse).
//
// TMEM: S_0 [0, 160), S_1 [160, 320), O [320, 448) + rounded-P row sum [448, 464).
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 2  // site numbers of the checked build

namespace mimo {

constexpr int kSwThreads = 448;
constexpr int kSwNMax = 160;
constexpr int kSwQBytes = 3 * 16384;                   // [128 rows][192 dims] as 3 boxes
constexpr int kSwKBox = kSwNMax * 128;                 // [N rows][64 dims], 1024-aligned
constexpr int kSwOffQ = 0;                             // 2 buffers
constexpr int kSwOffK = 2 * kSwQBytes;                 // 98304: 3 boxes
constexpr int kSwOffV = kSwOffK + 3 * kSwKBox;         // 2 boxes
constexpr int kSwOffOnes = kSwOffV + 2 * kSwKBox;      // the third value block: [N rows][64] ones
constexpr int kSwOffML = kSwOffOnes + kSwKBox;          // [2][128] float4 (m, l, sink term, -)
constexpr int kSwOffBar = kSwOffML + 2 * 128 * 16;
constexpr uint32_t kSwColO = 2 * kSwNMax, kSwColSum = kSwColO + 128;  // 320, 448
static_assert(kSwOffOnes % 1024 == 0 && kSwColSum + 16 <= 512, "SWA prefill layout");
constexpr int kSwSmemBytes = kSwOffBar + 256 + 1024;

struct SwaParams {
  const int32_t* cu_seqlens;
  const float* sinks;
  void* out;
  float* lse;
  int total, Hq, Hkv, G, QB, N, window;
  int num_seqs, max_seqlen, num_pairs, num_items;   // items = pairs of blocks
  float scale_log2, v_scale;
  int out_f32, out_v8;
};

// A work item is a pair of blocks: queries [q0, q0 + 2 QB) of one sequence.
struct SwItem {
  int b0, len, q0, g, nblk;  // nblk: 1 or 2 valid blocks
  bool valid;
};

__device__ __forceinline__ SwItem sw_decode(const SwaParams& p, int item) {
  SwItem it;
  const int per_qb = p.Hkv * p.num_seqs;
  const int qb = item / per_qb;
  const int rem = item % per_qb;
  const int seq = rem / p.Hkv;
  it.g = rem % p.Hkv;
  it.b0 = p.cu_seqlens[seq];
  it.len = p.cu_seqlens[seq + 1] - it.b0;
  it.q0 = qb * 2 * p.QB;
  it.valid = it.q0 < it.len;
  if (!seq_in_bounds(it.b0, it.len, p.max_seqlen, p.total)) {
    // a cu_seqlens entry out of order or past total_tokens, or a sequence
    // longer than max_seqlen: no row of it is read or written
    record_status(1 /* MIMO_ERR_INVALID_ARG */);
    it.valid = false;
  }
  it.nblk = (it.q0 + p.QB < it.len) ? 2 : 1;
  return it;
}

// First valid item at or after round r of this CTA (round-robin); -1 if none.
__device__ __forceinline__ int sw_next(const SwaParams& p, int r, int rounds, SwItem& it) {
  for (; r < rounds; ++r) {
    const int item = r * gridDim.x + blockIdx.x;
    if (item >= p.num_items) return -1;
    it = sw_decode(p, item);
    if (it.valid) return r;
  }
  return -1;
}

__global__ void __launch_bounds__(kSwThreads, 1)
    prefill_swa_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const SwaParams p) {
  extern __shared__ __align__(1024) uint8_t ssmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ssmem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSwOffBar);
  uint64_t* q_full = bars + 0;    // [2]
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* k_full = bars + 4;
  uint64_t* k_empty = bars + 5;
  uint64_t* v_full = bars + 6;
  uint64_t* v_empty = bars + 7;
  uint64_t* s_full = bars + 8;    // [2]
  uint64_t* p_full = bars + 10;   // [2]
  uint64_t* o_full = bars + 12;
  uint64_t* o_empty = bars + 13;
  uint64_t* ml_full = bars + 14;  // [2]
  uint64_t* ml_empty = bars + 16; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 19);
  uint64_t* mma_drain = bars + 20;  // teardown after a timed-out wait only
  volatile int* never_flag = reinterpret_cast<volatile int*>(bars + 21);  // never raised
  float4* ml = reinterpret_cast<float4*>(smem + kSwOffML);  // [2][128] (m, l, sink term) per row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // phases the producer armed: Q for blocks 0, 1, ... (buffer n & 1), K and V per pair
  int armed_q = 0, armed_k = 0, armed_v = 0;
  // the ones block, third 64-column block of the value operand: bf16 1.0
  for (int i = threadIdx.x; i < kSwKBox / 4; i += kSwThreads)
    reinterpret_cast<uint32_t*>(smem + kSwOffOnes)[i] = 0x3F803F80u;
  fence_proxy_async_smem();
  if (warp == 12) {
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&q_full[i], 1);
        mbar_init(&q_empty[i], 1);
        mbar_init(&s_full[i], 1);
        mbar_init(&p_full[i], 128);
        mbar_init(&ml_full[i], 128);
        mbar_init(&ml_empty[i], 128);
      }
      mbar_init(k_full, 1);
      mbar_init(k_empty, 1);
      mbar_init(v_full, 1);
      mbar_init(v_empty, 1);
      mbar_init(o_full, 1);
      mbar_init(o_empty, 128);
      mbar_init(mma_drain, 1);
      *never_flag = 0;
      *abort_flag = timed_out_before() ? 1 : 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  const int rounds = *abort_flag ? 0 : (p.num_items + gridDim.x - 1) / gridDim.x;
  const int N = p.N;

  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      auto load_q = [&](const SwItem& it, int blk, int b) {
        mbar_arrive_expect_tx(&q_full[b], kSwQBytes);
        ++armed_q;
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_3d(smem + kSwOffQ + b * kSwQBytes + c * 16384, &tm_q, &q_full[b], c * 64,
                      it.g * p.G, it.b0 + it.q0 + blk * p.QB);
      };
      // Blocks are numbered n = 0, 1, ... over this CTA's pairs; block n uses Q
      // buffer n & 1.  The pair's K/V window is loaded at its first block.
      SwItem cur, nxt;
      int r = sw_next(p, 0, rounds, cur);
      if (r >= 0) load_q(cur, 0, 0);
      bool ok = true;
      int n = 0, kp = 0;
      while (ok && r >= 0) {
        const int k0 = cur.q0 + 2 * p.QB - N;  // may be negative: zero-filled or masked
        int rn = -1;
        for (int blk = 0; ok && blk < cur.nblk; ++blk, ++n) {
          if (blk == 0) {
            if (kp >= 1 && !(ok = wait_bounded(k_empty, (kp - 1) & 1, abort_flag))) break;
            mbar_arrive_expect_tx(k_full, 3 * N * 128);
            ++armed_k;
#pragma unroll
            for (int c = 0; c < 3; ++c)
              tma_load_3d(smem + kSwOffK + c * kSwKBox, &tm_k, k_full, c * 64, cur.g, cur.b0 + k0);
          }
          // the next block's Q, one block ahead (its buffer was freed by S(n-1));
          // the next pair is looked up only now, after this pair's loads are out
          const int bn = (n + 1) & 1;
          const bool next_in_pair = (blk + 1 < cur.nblk);
          if (!next_in_pair) rn = sw_next(p, r + 1, rounds, nxt);
          if (next_in_pair || rn >= 0) {
            if (n + 1 >= 2 && !(ok = wait_bounded(&q_empty[bn], (((n + 1) >> 1) - 1) & 1, abort_flag))) break;
            if (next_in_pair)
              load_q(cur, blk + 1, bn);
            else
              load_q(nxt, 0, bn);
          }
          if (blk == 0) {
            if (kp >= 1 && !(ok = wait_bounded(v_empty, (kp - 1) & 1, abort_flag))) break;
            mbar_arrive_expect_tx(v_full, 2 * N * 128);
            ++armed_v;
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_load_3d(smem + kSwOffV + c * kSwKBox, &tm_v, v_full, c * 64, cur.g, cur.b0 + k0);
            ++kp;
          }
        }
        cur = nxt;
        r = rn;
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, N, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 144, false, true);  // 128 value dims + 16 ones
      const uint32_t tO = tbase + kSwColO;
      bool ok = true;
      // O = P(m) V over N keys: N/16 MMAs (P: 8 TMEM columns each; V: 16 rows = 2 KB).
      // Block m is the blk-th of pair kp_m; the pair's V is waited for at its first
      // block and released after its last.
      auto do_pv = [&](int m, int kp_m, bool first_of_pair, bool last_of_pair) {
        const int bm = m & 1;
        if (!(ok = wait_bounded(&p_full[bm], (m >> 1) & 1, abort_flag))) return;
        if (first_of_pair && !(ok = wait_bounded(v_full, kp_m & 1, abort_flag))) return;
        if (m >= 1 && !(ok = wait_bounded(o_empty, (m - 1) & 1, abort_flag))) return;
        tc_fence_after();
        const uint32_t tP = tbase + bm * kSwNMax;
        const uint32_t aV = sbase + kSwOffV;
        for (int kk = 0; kk < N / 16; ++kk)
          umma_ts(tO, tP + kk * 8, smem_desc_sw128(aV + kk * 2048, kSwKBox, 1024), idesc_o,
                  kk > 0 ? 1u : 0u);
        umma_commit(o_full);
        if (last_of_pair) umma_commit(v_empty);
      };
      SwItem it;
      int n = 0, kp = 0;
      int pm = -1, pkp = 0;     // previous block: number, pair
      bool pfirst = false, plast = false;
      for (int r = sw_next(p, 0, rounds, it); ok && r >= 0; r = sw_next(p, r + 1, rounds, it), ++kp) {
        for (int blk = 0; ok && blk < it.nblk; ++blk, ++n) {
          const int b = n & 1;
          if (!(ok = wait_bounded(&q_full[b], (n >> 1) & 1, abort_flag))) break;
          if (blk == 0 && !(ok = wait_bounded(k_full, kp & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t aQ = sbase + kSwOffQ + b * kSwQBytes;
          const uint32_t aK = sbase + kSwOffK;
          const uint32_t tS = tbase + b * kSwNMax;
#pragma unroll
          for (int kk = 0; kk < 12; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            umma_ss(tS, smem_desc_sw128(aQ + (kk >> 2) * 16384 + off, 16, 1024),
                    smem_desc_sw128(aK + (kk >> 2) * kSwKBox + off, 16, 1024), idesc_s,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[b]);
          umma_commit(&q_empty[b]);
          if (blk == it.nblk - 1) umma_commit(k_empty);
          if (pm >= 0) do_pv(pm, pkp, pfirst, plast);
          pm = n;
          pkp = kp;
          pfirst = (blk == 0);
          plast = (blk == it.nblk - 1);
        }
      }
      if (ok && pm >= 0) do_pv(pm, pkp, pfirst, plast);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int s = warp >> 2;                   // this warpgroup's blocks: n & 1 == s
    const int r = (warp & 3) * 32 + lane;      // TMEM lane = row = query * G + head
    const int a = r / p.G, hh = r % p.G;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    SwItem it;
    int n = 0;
    bool ok = true;
    for (int rr = sw_next(p, 0, rounds, it); ok && rr >= 0; rr = sw_next(p, rr + 1, rounds, it))
    for (int blk = 0; ok && blk < it.nblk; ++blk, ++n) {
      const int b = n & 1;
      if (b != s) continue;
      const int hg = it.g * p.G + hh;
      const int qpos = it.q0 + blk * p.QB + a;
      const int k0 = it.q0 + 2 * p.QB - N;
      const int c_hi = qpos - k0;                              // keys <= qpos
      const int c_lo = max(qpos - p.window + 1, 0) - k0;       // keys in window, >= 0
      const float sg2 = p.sinks ? p.sinks[hg] * 1.4426950408889634f : -INFINITY;
      if (!(ok = wait_bounded(&s_full[b], (n >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t tS = tbase + lane_off + b * kSwNMax;
      // pass 1: row max over the visible columns.  The row is read in chunks of
      // 48 columns (one wait per chunk); columns at or past N lie outside
      // [c_lo, c_hi] and are masked like the window's edges.
      float mx0 = -INFINITY, mx1 = -INFINITY;
      for (int c0 = 0; c0 < N; c0 += 48) {
        uint32_t v[48];
        tmem_load48_sync(tS + c0, v);
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          const int cq0 = c0 + 16 * q;
          if (cq0 >= c_lo && cq0 + 15 <= c_hi) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              mx0 = fmax3(mx0, __uint_as_float(v[16 * q + e]), __uint_as_float(v[16 * q + e + 1]));
              mx1 = fmax3(mx1, __uint_as_float(v[16 * q + e + 2]), __uint_as_float(v[16 * q + e + 3]));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = cq0 + e;
              if (c >= c_lo && c <= c_hi) mx0 = fmaxf(mx0, __uint_as_float(v[16 * q + e]));
            }
          }
        }
      }
      const float m = fmaxf(sg2, fmaxf(mx0, mx1) * p.scale_log2);
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      // pass 2: P = 2^(s*scale - m) (0 outside the window), bf16 over the same
      // columns (P of columns [c0, c0 + 48) lands in [c0 / 2, c0 / 2 + 24), behind
      // the read position).  The unrounded sum gives lse; the output's
      // normaliser, the sum of the rounded P, comes from the row-sum MMA.
      float2 l2 = make_float2(0.f, 0.f);
      for (int c0 = 0; c0 < N; c0 += 48) {
        uint32_t v[48];
        tmem_load48_sync(tS + c0, v);
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          const int cq0 = c0 + 16 * q;
          uint32_t pk[8];
          if (cq0 >= c_lo && cq0 + 15 <= c_hi) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 x = fma2(make_float2(__uint_as_float(v[16 * q + 2 * e]), __uint_as_float(v[16 * q + 2 * e + 1])),
                                    make_float2(p.scale_log2, p.scale_log2), make_float2(neg_m, neg_m));
              const float2 pe = make_float2(ex2(x.x), ex2(x.y));
              pk[e] = pack_bf16(pe.x, pe.y);
              l2 = add2(l2, pe);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = cq0 + 2 * e;
              const float x0 = fmaf(__uint_as_float(v[16 * q + 2 * e]), p.scale_log2, neg_m);
              const float x1 = fmaf(__uint_as_float(v[16 * q + 2 * e + 1]), p.scale_log2, neg_m);
              const float2 pe = make_float2((c >= c_lo && c <= c_hi) ? ex2(x0) : 0.f,
                                            (c + 1 >= c_lo && c + 1 <= c_hi) ? ex2(x1) : 0.f);
              pk[e] = pack_bf16(pe.x, pe.y);
              l2 = add2(l2, pe);
            }
          }
          if (cq0 < N) tmem_st8(tS + cq0 / 2, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
      const float ps = (p.sinks && m != -INFINITY) ? ex2(sg2 - m) : 0.f;  // the sink's term
      if (n >= 2 && !(ok = wait_bounded(&ml_empty[b], ((n >> 1) - 1) & 1, abort_flag))) break;
      ml[b * 128 + r] = make_float4(m, l2.x + l2.y + ps, ps, 0.f);
      mbar_arrive(&ml_full[b]);
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ epilogue
    const int r = threadIdx.x - 256;
    const int a = r / p.G, hh = r % p.G;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tbase + lane_off + kSwColO;
    SwItem it;
    int n = 0;
    bool ok = true;
    for (int rr = sw_next(p, 0, rounds, it); ok && rr >= 0; rr = sw_next(p, rr + 1, rounds, it))
    for (int blk = 0; ok && blk < it.nblk; ++blk, ++n) {
      const int b = n & 1;
      if (!(ok = wait_bounded(o_full, n & 1, abort_flag))) break;
      tc_fence_after();
      if (!(ok = wait_bounded(&ml_full[b], (n >> 1) & 1, abort_flag))) break;
      const float4 mlv = ml[b * 128 + r];  // m (base 2), unrounded sum with the sink, the sink's term
      mbar_arrive(&ml_empty[b]);
      float rs[16];
      tmem_load16_sync(tbase + lane_off + kSwColSum, rs);  // rounded-P row sum (16 equal columns)
      const float lr = rs[0] + mlv.z;
      const int qpos = it.q0 + blk * p.QB + a;
      const int hg = it.g * p.G + hh;
      const bool live =
          qpos < it.len && MIMO_ROW_OK((long long)(it.b0 + qpos) * p.Hq + hg, (long long)p.total * p.Hq);
      const int tok = it.b0 + qpos;
      const float f = (lr > 0.f) ? p.v_scale / lr : 0.f;
      const size_t ob = ((size_t)tok * p.Hq + hg) * 128;
      // O in two 64-column halves (registers: 448 threads leave 128 per thread);
      // O is released to the next P.V after the second half is in registers.
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float o[64];
        tmem_load64_sync(tO + h * 64, o);
        if (h == 1) {
          tc_fence_before();
          mbar_arrive(o_empty);
        }
        if (!live) continue;
        if (p.out_f32) {
          float* dst = reinterpret_cast<float*>(p.out) + ob + h * 64;
          if (p.out_v8) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              st_global_v8(dst + 8 * e, __float_as_uint(o[8 * e] * f), __float_as_uint(o[8 * e + 1] * f),
                           __float_as_uint(o[8 * e + 2] * f), __float_as_uint(o[8 * e + 3] * f),
                           __float_as_uint(o[8 * e + 4] * f), __float_as_uint(o[8 * e + 5] * f),
                           __float_as_uint(o[8 * e + 6] * f), __float_as_uint(o[8 * e + 7] * f));
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              reinterpret_cast<float4*>(dst)[e] =
                  make_float4(o[4 * e] * f, o[4 * e + 1] * f, o[4 * e + 2] * f, o[4 * e + 3] * f);
          }
        } else {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + ob + h * 64;
          if (p.out_v8) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              st_global_v8(dst + 16 * e, pack_bf16(o[16 * e + 0] * f, o[16 * e + 1] * f),
                           pack_bf16(o[16 * e + 2] * f, o[16 * e + 3] * f),
                           pack_bf16(o[16 * e + 4] * f, o[16 * e + 5] * f),
                           pack_bf16(o[16 * e + 6] * f, o[16 * e + 7] * f),
                           pack_bf16(o[16 * e + 8] * f, o[16 * e + 9] * f),
                           pack_bf16(o[16 * e + 10] * f, o[16 * e + 11] * f),
                           pack_bf16(o[16 * e + 12] * f, o[16 * e + 13] * f),
                           pack_bf16(o[16 * e + 14] * f, o[16 * e + 15] * f));
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              uint4 u;
              u.x = pack_bf16(o[8 * e + 0] * f, o[8 * e + 1] * f);
              u.y = pack_bf16(o[8 * e + 2] * f, o[8 * e + 3] * f);
              u.z = pack_bf16(o[8 * e + 4] * f, o[8 * e + 5] * f);
              u.w = pack_bf16(o[8 * e + 6] * f, o[8 * e + 7] * f);
              reinterpret_cast<uint4*>(dst)[e] = u;
            }
          }
        }
      }
      if (live && p.lse)
        p.lse[(size_t)hg * p.total + tok] =
            (mlv.y > 0.f) ? (mlv.x * 0.6931471805599453f + logf(mlv.y)) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // a role gave up: the loads and MMAs still in flight land before the CTA
    // frees its TMEM and exits
    if (warp == 12 && lane == 0) {
      drain_armed(&q_full[0], (armed_q + 1) / 2, never_flag);
      drain_armed(&q_full[1], armed_q / 2, never_flag);
      drain_armed(k_full, armed_k, never_flag);
      drain_armed(v_full, armed_v, never_flag);
    }
    if (warp == 13 && lane == 0 && rounds > 0) drain_mma(mma_drain, never_flag);  // rounds > 0: MMAs may have been issued
    __syncthreads();
  }
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace mimo
