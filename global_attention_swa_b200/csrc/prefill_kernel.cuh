// Prefill: packed variable-length causal GQA attention with a sliding window
// and a per-head attention sink, on 5th-generation tensor cores (tcgen05).
//
// MiMo-V2-Flash model doc, "Key features" (hybrid attention: 5:1 sliding
// window / global layers, small window, learnable attention-sink bias) and
// MiMoV2FlashConfig (64 query heads over 4 key/value heads, head_dim 192 for
// query/key, v_head_dim 128, sliding_window 129).
//
// Work item = one 128-query tile of one sequence x two query heads of the same
// key/value group.  Both heads see exactly the same key tiles, so each K/V
// tile staged in shared memory feeds two 128x128 score tiles.
//
// The kernel is persistent: one CTA per SM walks the item list (heaviest
// query tiles first, snake order across CTAs).  Barrier phases run on across
// items, so the next item's Q / K loads and first score MMAs overlap the
// current item's last P.V products and its epilogue.
//
//   warp 8      TMA producer: Q (2 x 48 KB), K ring (2 x 48 KB), V (32 KB);
//               also allocates / frees the 512 TMEM columns.
//   warp 9      MMA issuer (one thread):  S_i = Q_i K^T   (tcgen05, SS)
//                                         O_i += P_i V    (tcgen05, TS: P from TMEM)
//   warps 10-11 idle (they complete the third warpgroup)
//   warps 0-3   softmax + epilogue of head 0 (TMEM lanes 0..127, one row each)
//   warps 4-7   softmax + epilogue of head 1
//
// Registers: launched at 168 per thread (384 threads); the producer/MMA
// warpgroup gives back down to 104 and the two softmax warpgroups take 200
// (2*128*200 + 128*104 = 64512 = 384*168; per SM sub-partition
// 200 + 200 + 104 registers x 32 lanes = 16128 <= 16384).
//
// TMEM columns: S_0 [0,128)  S_1 [128,256)  O_0 [256,384)  O_1 [384,512).
// P_i (bf16, two per 32-bit column) overwrites the first 64 columns of S_i.
//
// Online softmax in base 2 with the sink folded into the running state:
// m starts at sigma_h*log2(e) and l at 1 (the sink's own term), so the sink
// enters the normaliser once and never the output.  The reference m is not
// the running max: P = 2^(s*scale - m) is computed against it as it stands,
// and it is moved to the row max (with O and l rescaled) only when a tile's
// sum of P leaves the range where fp32 and bf16 hold it (above 2^64, or NaN
// from an overflow), or a row without a sink has no reference yet.  That is
// exact, because O and l share the reference, and the relative precision of
// bf16 P and of the fp32 sums does not depend on their scale.  The common
// path therefore does no row-max pass at all.
//
// Key tiles wholly outside [q0 - window + 1, q0 + 127] are never loaded: a
// 129-wide window touches at most two 128-key tiles per query tile.
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 1  // site numbers of the checked build

namespace mimo {

constexpr int kPfThreads = 384;
constexpr int kPfTile = 128;
constexpr int kPfQBytes = 128 * 192 * 2;  // 49152: 3 boxes of [128 rows][64 dims]
constexpr int kPfKBytes = 128 * 192 * 2;  // 49152
constexpr int kPfVBytes = 128 * 128 * 2;  // 32768: 2 boxes of [128 keys][64 dims]
constexpr int kPfOffQ0 = 0;
constexpr int kPfOffQ1 = kPfQBytes;
constexpr int kPfOffK = 2 * kPfQBytes;                 // 2 stages
constexpr int kPfOffV = kPfOffK + 2 * kPfKBytes;       // 196608
constexpr int kPfOffBar = kPfOffV + kPfVBytes;         // 229376
constexpr int kPfSmemBytes = kPfOffBar + 256 + 1024;   // barriers + alignment slack

struct PrefillParams {
  const int32_t* cu_seqlens;  // [num_seqs + 1]
  const float* sinks;         // [Hq] or null
  void* out;                  // [total, Hq, 128]
  float* lse;                 // [Hq, total] or null
  int total, Hq, Hkv, G;
  int window;
  int pairs_per_group;        // ceil(G / 2)
  int num_seqs;
  int max_seqlen;
  int num_qtiles;             // ceil(max_seqlen / 128)
  int num_items;              // num_qtiles * Hkv * pairs_per_group * num_seqs
  float scale_log2;           // softmax_scale * log2(e)
  float v_scale;
  int out_f32;
  int out_v8;                 // out is 32-byte aligned: one full sector per store
};

// K-major operand (rows of 64 bf16 = 128 B, 8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  return smem_desc_sw128(addr, 16, 1024);
}
// MN-major operand V: 64-column atoms 16 KB apart (LBO), 8-key groups 1024 B apart (SBO).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr) {
  return smem_desc_sw128(addr, 16384, 1024);
}

// One work item, decoded.  Items are numbered heaviest query tile first;
// within a query tile, sequence then key/value head pair, so that a
// sequence's items sit together: in a pack of mixed lengths, where the long
// sequences alone have the high query tiles, this spreads the work evenly
// over the CTAs' round-robin shares (busiest CTA 1.04x the mean for 16
// sequences of 512..8192 tokens, against 1.41x with the sequence innermost).
struct PfItem {
  int b0, len, q0, g, h0, j_lo, n_kt;
  bool has1, valid;
};

__device__ __forceinline__ int pf_item_index(int round, int cta, int ctas) {
  return round * ctas + ((round & 1) ? (ctas - 1 - cta) : cta);  // snake order
}

__device__ __forceinline__ PfItem pf_decode(const PrefillParams& p, int item) {
  PfItem it;
  const int per_q = p.Hkv * p.pairs_per_group * p.num_seqs;
  const int qt = p.num_qtiles - 1 - item / per_q;
  const int rem = item % per_q;
  const int npairs = p.Hkv * p.pairs_per_group;
  const int seq = rem / npairs;
  const int pair = rem % npairs;
  it.g = pair / p.pairs_per_group;
  const int pp = pair % p.pairs_per_group;
  it.h0 = it.g * p.G + 2 * pp;
  it.has1 = (2 * pp + 1) < p.G;
  it.b0 = p.cu_seqlens[seq];
  it.len = p.cu_seqlens[seq + 1] - it.b0;
  it.q0 = qt * kPfTile;
  it.valid = it.q0 < it.len;
  if (!seq_in_bounds(it.b0, it.len, p.max_seqlen, p.total)) {
    // a cu_seqlens entry out of order or past total_tokens, or a sequence
    // longer than max_seqlen: no row of it is read or written
    record_status(1 /* MIMO_ERR_INVALID_ARG */);
    it.valid = false;
  }
  if (it.valid) {
    const int last_q = min(it.q0 + kPfTile - 1, it.len - 1);
    const int j_hi = last_q / kPfTile;
    it.j_lo = p.window > 0 ? max(0, it.q0 - p.window + 1) / kPfTile : 0;
    it.n_kt = j_hi - it.j_lo + 1;
  } else {
    it.j_lo = 0;
    it.n_kt = 0;
  }
  return it;
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t psmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(psmem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPfOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;   // [2]
  uint64_t* k_empty = bars + 4;  // [2]
  uint64_t* v_full = bars + 6;
  uint64_t* v_empty = bars + 7;
  uint64_t* s_full = bars + 8;   // [2]
  uint64_t* p_full = bars + 10;  // [2]
  uint64_t* o_full = bars + 12;  // [2]
  uint64_t* o_empty = bars + 14; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 17);
  uint64_t* mma_drain = bars + 18;  // teardown after a timed-out wait only
  volatile int* never_flag = reinterpret_cast<volatile int*>(bars + 19);  // never raised
  // for the teardown, kept here rather than in registers the loops carry: the
  // phases the producer armed on q_full, on the K ring (tiles in order) and on
  // v_full, and whether the MMA thread had work
  int* armed = reinterpret_cast<int*>(bars + 20);  // [4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 8) {
    if (lane == 0) {
      mbar_init(q_full, 1);
      mbar_init(q_empty, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&k_full[i], 1);
        mbar_init(&k_empty[i], 1);
        mbar_init(&s_full[i], 1);
        mbar_init(&p_full[i], 128);
        mbar_init(&o_full[i], 1);
        mbar_init(&o_empty[i], 128);
      }
      mbar_init(v_full, 1);
      mbar_init(v_empty, 1);
      mbar_init(mma_drain, 1);
      *never_flag = 0;
      armed[0] = armed[1] = armed[2] = armed[3] = 0;
      // sampled once, so every thread of the CTA sees the same decision
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
  // after a recorded timeout elsewhere, do no work (but still free TMEM)
  const int rounds = *abort_flag ? 0 : (p.num_items + gridDim.x - 1) / gridDim.x;

  if (warp >= 8) {
    setmaxnreg_dec<104>();
  }
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int n = 0;   // items loaded
      int kt = 0;  // key tiles loaded (all items)
      bool ok = true;
      for (int r = 0; ok && r < rounds; ++r) {
        const int item = pf_item_index(r, blockIdx.x, gridDim.x);
        if (item >= p.num_items) continue;
        const PfItem it = pf_decode(p, item);
        if (!it.valid) continue;
        // Q buffer is free once the previous item's last score MMA completed
        if (n > 0 && !(ok = wait_bounded(q_empty, (n - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, it.has1 ? 2 * kPfQBytes : kPfQBytes);
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_3d(smem + kPfOffQ0 + c * 16384, &tm_q, q_full, c * 64, it.h0, it.b0 + it.q0);
        if (it.has1) {
#pragma unroll
          for (int c = 0; c < 3; ++c)
            tma_load_3d(smem + kPfOffQ1 + c * 16384, &tm_q, q_full, c * 64, it.h0 + 1, it.b0 + it.q0);
        }
        for (int t = 0; t < it.n_kt; ++t, ++kt) {
          const int row = it.b0 + (it.j_lo + t) * kPfTile;
          const int ks = kt & 1;
          if (kt >= 2 && !(ok = wait_bounded(&k_empty[ks], ((kt >> 1) - 1) & 1, abort_flag))) break;
          mbar_arrive_expect_tx(&k_full[ks], kPfKBytes);
          armed[1] = kt + 1;
#pragma unroll
          for (int c = 0; c < 3; ++c)
            tma_load_3d(smem + kPfOffK + ks * kPfKBytes + c * 16384, &tm_k, &k_full[ks], c * 64, it.g, row);
          if (kt >= 1 && !(ok = wait_bounded(v_empty, (kt - 1) & 1, abort_flag))) break;
          mbar_arrive_expect_tx(v_full, kPfVBytes);
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d(smem + kPfOffV + c * 16384, &tm_v, v_full, c * 64, it.g, row);
        }
        ++n;
      }
      // every item counted in n had its Q armed; V is armed for tiles [0, kt)
      armed[0] = n;
      armed[2] = kt;
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      armed[3] = rounds > 0;
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      const uint32_t tS0 = tbase + 0, tS1 = tbase + 128, tO0 = tbase + 256, tO1 = tbase + 384;
      // Descriptors as one shared high word plus a low word per operand; the
      // per-MMA offsets below are compile-time constants (address units of 16 B).
      constexpr uint32_t dhi = desc_hi_sw128(1024);
      const uint32_t dQ0 = desc_lo_sw128(sbase + kPfOffQ0, 16), dQ1 = desc_lo_sw128(sbase + kPfOffQ1, 16);
      const uint32_t dK0 = desc_lo_sw128(sbase + kPfOffK, 16);
      const uint32_t dV = desc_lo_sw128(sbase + kPfOffV, 16384);
      // S_i = Q_i K^T over 192 dims = 12 MMAs of K=16 (3 swizzle boxes x 4 steps of 32 B)
      auto issue_s = [&](uint32_t tS, uint32_t dQ, uint32_t dK) {
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss_lo(tS, dQ + off, dK + off, dhi, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_i += P_i V over 128 keys = 8 MMAs of K=16 (P: 8 TMEM columns each; V: 16 rows = 2 KB)
      auto issue_pv = [&](uint32_t tO, uint32_t tP, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts_lo(tO, tP + kk * 8, dV + ((kk * 2048) >> 4), dhi, idesc_o, (acc || kk > 0) ? 1u : 0u);
      };
      auto dK = [&](int stage) { return dK0 + static_cast<uint32_t>(stage) * (kPfKBytes >> 4); };
      int n = 0;           // items
      int n1 = 0;          // items with a second head
      int kt = 0;          // key tiles (all items): K ring and V phases
      int t0 = 0, t1 = 0;  // score tiles of head 0 / head 1: s_full / p_full phases
      bool ok = true;
      for (int r = 0; ok && r < rounds; ++r) {
        const int item = pf_item_index(r, blockIdx.x, gridDim.x);
        if (item >= p.num_items) continue;
        const PfItem it = pf_decode(p, item);
        if (!it.valid) continue;
        if (!(ok = wait_bounded(q_full, n & 1, abort_flag))) break;
        if (!(ok = wait_bounded(&k_full[kt & 1], (kt >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        {
          issue_s(tS0, dQ0, dK(kt & 1));
          umma_commit(&s_full[0]);
          if (it.has1) {
            issue_s(tS1, dQ1, dK(kt & 1));
            umma_commit(&s_full[1]);
          }
          umma_commit(&k_empty[kt & 1]);
          if (it.n_kt == 1) umma_commit(q_empty);
        }
        for (int t = 0; t < it.n_kt; ++t, ++kt) {
          const bool last = (t == it.n_kt - 1);
          if (!(ok = wait_bounded(v_full, kt & 1, abort_flag))) break;
          if (!(ok = wait_bounded(&p_full[0], t0 & 1, abort_flag))) break;
          // O_0 is free once the previous item's epilogue has read it
          if (t == 0 && n > 0 && !(ok = wait_bounded(&o_empty[0], (n - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(tO0, tS0, t > 0);
          ++t0;
          if (last) umma_commit(&o_full[0]);
          const int kn = kt + 1;
          if (!last) {
            if (!(ok = wait_bounded(&k_full[kn & 1], (kn >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_s(tS0, dQ0, dK(kn & 1));
            umma_commit(&s_full[0]);
            if (!it.has1 && t + 1 == it.n_kt - 1) umma_commit(q_empty);
          }
          if (it.has1) {
            if (!(ok = wait_bounded(&p_full[1], t1 & 1, abort_flag))) break;
            if (t == 0 && n1 > 0 && !(ok = wait_bounded(&o_empty[1], (n1 - 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(tO1, tS1, t > 0);
            ++t1;
            if (last) umma_commit(&o_full[1]);
          }
          umma_commit(v_empty);
          if (!last) {
            if (it.has1) {
              issue_s(tS1, dQ1, dK(kn & 1));
              umma_commit(&s_full[1]);
              if (t + 1 == it.n_kt - 1) umma_commit(q_empty);
            }
            umma_commit(&k_empty[kn & 1]);
          }
        }
        ++n;
        if (it.has1) ++n1;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / epilogue
    setmaxnreg_inc<200>();
    const int i = warp >> 2;  // which head of the pair
    const int r = threadIdx.x & 127;  // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + i * 128;
    const uint32_t tO = tbase + lane_off + 256 + i * 128;
    int n = 0;   // items this head slot took part in
    int tg = 0;  // score tiles this head slot consumed
    bool ok = true;
    for (int rr = 0; ok && rr < rounds; ++rr) {
      const int item = pf_item_index(rr, blockIdx.x, gridDim.x);
      if (item >= p.num_items) continue;
      const PfItem it = pf_decode(p, item);
      if (!it.valid || (i == 1 && !it.has1)) continue;
      const int h = it.h0 + i;
      const int qpos = it.q0 + r;
      const float sg2 = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
      float m = sg2;
      float l = p.sinks ? 1.f : 0.f;   // exact row sum (lse)
      float lr = l;                    // sum of the bf16-rounded P that enter P.V (output)
      for (int t = 0; t < it.n_kt; ++t, ++tg) {
        const int kpos0 = (it.j_lo + t) * kPfTile;
        if (!(ok = wait_bounded(&s_full[i], tg & 1, abort_flag))) break;
        tc_fence_after();
        float s[128];
        tmem_load128_sync(tS, s);
        const bool full_tile = (kpos0 + kPfTile - 1 <= it.q0) &&
                               (p.window == 0 || (it.q0 + kPfTile - 1) - kpos0 <= p.window - 1);
        if (!full_tile) {
          const int hi_k = qpos - kpos0;                                  // keys <= hi_k visible
          const int lo_k = p.window > 0 ? qpos - p.window + 1 - kpos0 : -1;  // keys >= lo_k visible
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = (c <= hi_k && c >= lo_k) ? s[c] : -INFINITY;
        }
        // Moves the reference m up to the row max of this tile where need is
        // set (rescaling l, lr and, on later tiles, O by 2^(m_old - m_new)).
        // The whole warp takes part: the O rescale is a warp-wide TMEM access.
        auto move_max = [&](bool need) {
          float mx8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; ++c) mx8[c & 7] = fmax3(mx8[c & 7], s[2 * c], s[2 * c + 1]);
          const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                 fmaxf(mx8[6], mx8[7]));
          const float m_new = fmaxf(m, mx * p.scale_log2);
          float alpha = 1.f;
          bool rescale_o = false;
          if (need && m_new > m) {
            alpha = ex2(m - m_new);  // 0 when m was -inf
            l *= alpha;
            lr *= alpha;
            m = m_new;
            rescale_o = (t > 0);
          }
          // O of the previous tile is complete here: S_i(t) was committed after PV_i(t-1).
          if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_load32_sync(tO + c * 32, o);
              const float a_ = rescale_o ? alpha : 1.f;
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a_);
              tmem_st32(tO + c * 32, o);
            }
          }
        };
        // P = 2^(s*scale - m), rounded to bf16 for the PV product, written over
        // the first 64 columns of S.  Two row sums: the unrounded values (lse,
        // exact to fp32) and the rounded ones, which normalise the output, so
        // that out = sum_j P~_j v_j / (sum_j P~_j + sink) weights the value rows
        // by exactly the P that multiplied them.
        float2 a, ar;
        auto exps = [&]() {
          const float neg_m = (m == -INFINITY) ? 0.f : -m;
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 nm2 = make_float2(neg_m, neg_m);
          float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          float2 acr[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float2 x = fma2(make_float2(s[64 * half + 2 * c], s[64 * half + 2 * c + 1]), sc2, nm2);
              const float2 e = make_float2(ex2(x.x), ex2(x.y));
              pk[c] = pack_bf16(e.x, e.y);
              acc[c & 1] = add2(acc[c & 1], e);
              add_bf16x2(acr[c & 1], pk[c]);
            }
            tmem_st32(tS + 32 * half, pk);
          }
          a = add2(acc[0], acc[1]);
          ar = add2(acr[0], acr[1]);
        };
        // The reference m is the sink's logit (or, with no sink, the first row
        // max), moved only when this tile's P would leave the safe range: P is
        // scale-free in bf16 and fp32, so the only hazards are overflow (a sum
        // above 2^64) and a row with no reference yet.
        if (__any_sync(0xffffffffu, m == -INFINITY)) move_max(m == -INFINITY);
        exps();
        const auto unsafe = [&]() { return !(a.x + a.y <= 0x1p64f); };  // also NaN
        if (__any_sync(0xffffffffu, unsafe())) {
          move_max(unsafe());
          tmem_wait_st();  // the first P stores are complete before they are overwritten
          exps();
        }
        l += a.x + a.y;
        lr += ar.x + ar.y;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[i]);
      }
      if (!ok) break;
      // ---------------- epilogue: O / l -> out, lse.  O is read out of TMEM
      // first and released, so the next item's P.V can start at once.
      if (!(ok = wait_bounded(&o_full[i], n & 1, abort_flag))) break;
      tc_fence_after();
      float o[128];
      tmem_load128_sync(tO, o);
      tc_fence_before();
      mbar_arrive(&o_empty[i]);
      ++n;
      if (qpos < it.len && MIMO_ROW_OK((long long)(it.b0 + qpos) * p.Hq + h, (long long)p.total * p.Hq)) {
        const int tok = it.b0 + qpos;
        const float f = (lr > 0.f) ? p.v_scale / lr : 0.f;
        const size_t ob = ((size_t)tok * p.Hq + h) * 128;
        if (p.out_f32) {
          float* dst = reinterpret_cast<float*>(p.out) + ob;
          if (p.out_v8) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              st_global_v8(dst + 8 * e, __float_as_uint(o[8 * e] * f), __float_as_uint(o[8 * e + 1] * f),
                           __float_as_uint(o[8 * e + 2] * f), __float_as_uint(o[8 * e + 3] * f),
                           __float_as_uint(o[8 * e + 4] * f), __float_as_uint(o[8 * e + 5] * f),
                           __float_as_uint(o[8 * e + 6] * f), __float_as_uint(o[8 * e + 7] * f));
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              reinterpret_cast<float4*>(dst)[e] =
                  make_float4(o[4 * e] * f, o[4 * e + 1] * f, o[4 * e + 2] * f, o[4 * e + 3] * f);
          }
        } else if (p.out_v8) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + ob;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_global_v8(dst + 16 * e, pack_bf16(o[16 * e + 0] * f, o[16 * e + 1] * f),
                         pack_bf16(o[16 * e + 2] * f, o[16 * e + 3] * f),
                         pack_bf16(o[16 * e + 4] * f, o[16 * e + 5] * f),
                         pack_bf16(o[16 * e + 6] * f, o[16 * e + 7] * f),
                         pack_bf16(o[16 * e + 8] * f, o[16 * e + 9] * f),
                         pack_bf16(o[16 * e + 10] * f, o[16 * e + 11] * f),
                         pack_bf16(o[16 * e + 12] * f, o[16 * e + 13] * f),
                         pack_bf16(o[16 * e + 14] * f, o[16 * e + 15] * f));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            uint4 u;
            u.x = pack_bf16(o[8 * e + 0] * f, o[8 * e + 1] * f);
            u.y = pack_bf16(o[8 * e + 2] * f, o[8 * e + 3] * f);
            u.z = pack_bf16(o[8 * e + 4] * f, o[8 * e + 5] * f);
            u.w = pack_bf16(o[8 * e + 6] * f, o[8 * e + 7] * f);
            dst[e] = u;
          }
        }
        if (p.lse)
          p.lse[(size_t)h * p.total + tok] = (l > 0.f) ? (m * 0.6931471805599453f + logf(l)) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // a role gave up: the loads and MMAs still in flight land before the CTA
    // frees its TMEM and exits
    if (warp == 8 && lane == 0) {
      drain_armed(q_full, armed[0], never_flag);
      drain_armed(&k_full[0], (armed[1] + 1) / 2, never_flag);
      drain_armed(&k_full[1], armed[1] / 2, never_flag);
      drain_armed(v_full, armed[2], never_flag);
    }
    if (warp == 9 && lane == 0 && armed[3]) drain_mma(mma_drain, never_flag);  // MMAs may have been issued
    __syncthreads();
  }
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace mimo
