// Prefill on CTA pairs: causal GQA attention with an optional window and a
// per-head attention sink, with tcgen05 MMAs of M = 256 issued for two CTAs
// (cta_group::2).
//
// MiMo-V2-Flash model doc, "Key features" (hybrid attention: 5:1 sliding
// window / global layers, learnable attention-sink bias) and MiMoV2FlashConfig
// (64 query heads over 4 key/value heads, head_dim 192, v_head_dim 128).
//
// A cluster of two CTAs works on one 128-query tile of one sequence x four
// query heads of one key/value group; CTA r holds heads h0 + 2r and
// h0 + 2r + 1 ("slot" 0 and 1).  Slot i of both CTAs forms one M = 256 MMA:
//   S_i  = Q_i K^T   (SS; A: each CTA's Q_i, B: K, 64 keys of it in each CTA)
//   O_i += P_i V     (SS; A: each CTA's P_i tile, B: V, 64 value dims in each CTA)
// so each CTA stages only half of every K and V tile.  That leaves room for a
// P tile per slot in shared memory: the next score tile of a slot is issued as
// soon as its softmax holds the current scores in registers, and the tensor
// pipe runs  S_0(t+1), S_1(t+1), P_0(t) V, P_1(t) V  per key tile while the
// softmax warps compute the exponentials of tile t+1.
//
//   warp 8      TMA producer of this CTA's Q_0, Q_1 and half K tiles
//   warp 9      score-MMA issuer (one thread, leader CTA only)
//   warp 10     TMA producer of this CTA's half V tiles
//   warp 11     P.V-MMA issuer (one thread, leader CTA only)
//   warps 0-3   softmax + epilogue of slot 0 (TMEM lanes 0..127, one row each)
//   warps 4-7   softmax + epilogue of slot 1
//
// Registers: launched at 168 per thread (384 threads); the producer / MMA
// warpgroup gives back down to 120 and the two softmax warpgroups take 192
// (2*128*192 + 128*120 = 64512 = 384*168).
//
// Shared memory per CTA: Q_0, Q_1 (48 KB each), P_0, P_1 (32 KB each), the K
// half tile (24 KB, one stage: the score stream has slack for its load),
// V half tiles in two stages (16 KB each: the P.V stream has none).  TMEM per CTA:
// S_0 [0,128)  S_1 [128,256)  O_0 [256,384)  O_1 [384,512).
//
// Barriers: loads are counted on the leader's full barriers (the leader's
// producer expects the bytes of both CTAs); MMA completions arrive on both
// CTAs' barriers (commit with a CTA mask); each softmax / epilogue warp of both
// CTAs arrives once (one lane, after every lane fenced its own accesses and
// the warp synchronised) on the leader's barriers.  The softmax is the one of the
// single-CTA kernel (prefill_kernel.cuh): base 2, the sink folded into the
// running max and sum, conditional rescaling of O, the output normalised by
// the sum of the bf16-rounded P.  Every wait is bounded.
#pragma once

#include "common.cuh"
#include "prefill_kernel.cuh"

namespace mimo {

constexpr int kPpThreads = 384;
constexpr int kPpQBytes = 128 * 192 * 2;        // 3 boxes of [128 rows][64 dims]
constexpr int kPpPBytes = 128 * 128 * 2;        // 2 boxes of [128 rows][64 keys]
constexpr int kPpKBytes = 64 * 192 * 2;         // 3 boxes of [64 keys][64 dims]
constexpr int kPpVBytes = 128 * 64 * 2;         // 1 box of [128 keys][64 dims]
constexpr int kPpOffQ = 0;                      // Q_0, Q_1
constexpr int kPpOffP = 2 * kPpQBytes;          // 98304: P_0, P_1
constexpr int kPpOffK = kPpOffP + 2 * kPpPBytes;  // 163840: one stage
constexpr int kPpOffV = kPpOffK + kPpKBytes;      // 188416: 2 stages
constexpr int kPpOffBar = kPpOffV + 2 * kPpVBytes;  // 221184
constexpr int kPpSmemBytes = kPpOffBar + 256 + 1024;

struct PairParams {
  const int32_t* cu_seqlens;
  const float* sinks;
  void* out;
  float* lse;
  int total, Hq, Hkv, G, window;
  int quads_per_group;  // G / 4
  int num_seqs, max_seqlen, num_qtiles, num_items;
  float scale_log2, v_scale;
  int out_f32, out_v8;
};

struct PpItem {
  int b0, len, q0, g, h0, j_lo, n_kt;
  bool valid;
};

// Items are numbered heaviest query tile first; within a query tile, head
// quad then sequence.  Both CTAs of a pair decode the same item.
__device__ __forceinline__ PpItem pp_decode(const PairParams& p, int item) {
  PpItem it;
  const int per_q = p.Hkv * p.quads_per_group * p.num_seqs;
  const int qt = p.num_qtiles - 1 - item / per_q;
  const int rem = item % per_q;
  const int seq = rem % p.num_seqs;
  const int quad = rem / p.num_seqs;
  it.g = quad / p.quads_per_group;
  it.h0 = it.g * p.G + 4 * (quad % p.quads_per_group);
  it.b0 = p.cu_seqlens[seq];
  it.len = p.cu_seqlens[seq + 1] - it.b0;
  it.q0 = qt * kPfTile;
  it.valid = it.q0 < it.len;
  if (!seq_in_bounds(it.b0, it.len, p.max_seqlen, p.total)) {
    record_status(1 /* MIMO_ERR_INVALID_ARG */);
    it.valid = false;
  }
  if (it.valid) {
    const int last_q = min(it.q0 + kPfTile - 1, it.len - 1);
    it.j_lo = p.window > 0 ? max(0, it.q0 - p.window + 1) / kPfTile : 0;
    it.n_kt = last_q / kPfTile - it.j_lo + 1;
  } else {
    it.j_lo = 0;
    it.n_kt = 0;
  }
  return it;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPpThreads, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const PairParams p) {
  extern __shared__ __align__(1024) uint8_t ppsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ppsmem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPpOffBar);
  // leader-side (arrivals / bytes of both CTAs counted there)
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 2;    // [2]
  uint64_t* s_free = bars + 4;    // [2] slot i's softmax of both CTAs read S_i
  uint64_t* p_full = bars + 6;    // [2] slot i's P tiles of both CTAs written
  uint64_t* o_empty = bars + 8;   // [2] slot i's O read by both epilogues
  // both CTAs (MMA completions, committed with CTA mask 0b11)
  uint64_t* q_empty = bars + 10;
  uint64_t* k_empty = bars + 11;
  uint64_t* v_empty = bars + 12;  // [2]
  uint64_t* s_full = bars + 14;   // [2]
  uint64_t* pv_done = bars + 16;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 19);
  volatile int* abort_seen = reinterpret_cast<volatile int*>(bars + 20);  // [2] per CTA rank

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint16_t kBoth = 0x3;

  if (warp == 8) {
    if (lane == 0) {
      mbar_init(q_full, 1);
      mbar_init(k_full, 1);
      mbar_init(q_empty, 1);
      mbar_init(k_empty, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&v_full[i], 1);
        mbar_init(&v_empty[i], 1);
        mbar_init(&s_free[i], 8);   // one elected lane per softmax warp of both CTAs
        mbar_init(&p_full[i], 8);   // one elected lane per softmax warp of both CTAs
        mbar_init(&o_empty[i], 8);   // one elected lane per softmax warp of both CTAs
        mbar_init(&s_full[i], 1);
        mbar_init(&pv_done[i], 1);
      }
      fence_mbar_init();
    }
  }
  cluster_sync();  // both CTAs running, their barriers initialised
  if (warp == 8) {
    // the same warp of both CTAs allocates for the pair (the address lands in both)
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 0) {
    // both CTAs take the same decision: each publishes its own reading of the
    // device status word to both CTAs, and both act on the union
    const uint32_t seen = timed_out_before() ? 1u : 0u;
    for (uint32_t r = 0; r < 2; ++r)
      st_shared_cluster_u32(mapa_shared(smem_u32((const void*)&abort_seen[rank]), r), seen);
  }
  tc_fence_before();
  cluster_sync();  // TMEM allocated, abort readings exchanged
  tc_fence_after();
  if (threadIdx.x == 0) *abort_flag = (abort_seen[0] | abort_seen[1]) ? 1 : 0;
  __syncthreads();
  const uint32_t tbase = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  const int nclusters = gridDim.x / 2, cl = blockIdx.x / 2;
  const int rounds = *abort_flag ? 0 : (p.num_items + nclusters - 1) / nclusters;
  // the leader's barriers, as shared::cluster addresses
  auto lead = [&](const uint64_t* b) { return mapa_shared(smem_u32(b), 0); };

  if (warp >= 8) setmaxnreg_dec<120>();
  if (warp == 10) {
    // ------------------------------------------------------------ V producer (each CTA)
    // Apart from the Q / K producer so that waiting for the single V buffer
    // never holds back the next key tile's K.
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      const uint32_t bv0 = lead(&v_full[0]), bv1 = lead(&v_full[1]);
      int kt = 0;
      bool ok = true;
      for (int r = 0; ok && r < rounds; ++r) {
        const int item = pf_item_index(r, cl, nclusters);
        if (item >= p.num_items) continue;
        const PpItem it = pp_decode(p, item);
        if (!it.valid) continue;
        for (int t = 0; t < it.n_kt; ++t, ++kt) {
          const int vs = kt & 1;
          if (kt >= 2 && !(ok = wait_bounded(&v_empty[vs], ((kt >> 1) - 1) & 1, abort_flag))) break;
          if (rank == 0) mbar_arrive_expect_tx(&v_full[vs], 2 * kPpVBytes);
          tma_load_3d_pair(smem + kPpOffV + vs * kPpVBytes, &tm_v, vs ? bv1 : bv0, 64 * (int)rank, it.g,
                           it.b0 + (it.j_lo + t) * kPfTile);
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ Q / K producer (each CTA)
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      const uint32_t bq = lead(q_full), bk = lead(k_full);
      int n = 0, kt = 0;
      bool ok = true;
      for (int r = 0; ok && r < rounds; ++r) {
        const int item = pf_item_index(r, cl, nclusters);
        if (item >= p.num_items) continue;
        const PpItem it = pp_decode(p, item);
        if (!it.valid) continue;
        if (n > 0 && !(ok = wait_bounded(q_empty, (n - 1) & 1, abort_flag))) break;
        if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * 2 * kPpQBytes);
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
          for (int c = 0; c < 3; ++c)
            tma_load_3d_pair(smem + kPpOffQ + s * kPpQBytes + c * 16384, &tm_q, bq, c * 64,
                             it.h0 + 2 * (int)rank + s, it.b0 + it.q0);
        for (int t = 0; t < it.n_kt; ++t, ++kt) {
          const int row = it.b0 + (it.j_lo + t) * kPfTile;
          if (kt >= 1 && !(ok = wait_bounded(k_empty, (kt - 1) & 1, abort_flag))) break;
          if (rank == 0) mbar_arrive_expect_tx(k_full, 2 * kPpKBytes);
#pragma unroll
          for (int c = 0; c < 3; ++c)
            tma_load_3d_pair(smem + kPpOffK + c * 8192, &tm_k, bk, c * 64, it.g, row + 64 * (int)rank);
          if (t == 0) {
            // with the item's first loads out, bring the next item's Q into L2,
            // so that its load after this item's last score tile skips DRAM
            for (int r2 = r + 1; r2 < rounds; ++r2) {
              const int item2 = pf_item_index(r2, cl, nclusters);
              if (item2 >= p.num_items) continue;
              const PpItem nx = pp_decode(p, item2);
              if (!nx.valid) continue;
#pragma unroll
              for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int c = 0; c < 3; ++c)
                  tma_prefetch_l2_3d(&tm_q, c * 64, nx.h0 + 2 * (int)rank + s, nx.b0 + nx.q0);
              break;
            }
          }
        }
        ++n;
      }
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------ MMA issuers (leader)
    // Two threads feed the tensor pipe: warp 9 issues the score products, warp
    // 11 the P.V products.  The two streams never touch the same TMEM columns
    // or shared memory (S_i vs O_i; Q, K vs P, V), so neither needs the other's
    // order, and while one waits on a barrier the other keeps the pipe busy (an
    // issuing thread advances only as fast as the pipe takes its MMAs).
    if (lane == 0 && rank == 0) {
      constexpr uint32_t dhi = desc_hi_sw128(1024);
      if (warp == 9) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(256, 128, false, false);
        const uint32_t dQ0 = desc_lo_sw128(sbase + kPpOffQ, 16);
        const uint32_t dK0 = desc_lo_sw128(sbase + kPpOffK, 16);
        // S_i = Q_i K^T: 12 K-steps of 16 dims (A boxes 16 KB apart, B boxes 8 KB apart)
        auto issue_s = [&](int i) {
          const uint32_t a = dQ0 + static_cast<uint32_t>(i) * (kPpQBytes >> 4);
          const uint32_t b = dK0;
          const uint32_t d = tbase + static_cast<uint32_t>(i) * 128;
#pragma unroll
          for (int kk = 0; kk < 12; ++kk)
            umma_ss_lo_pair(d, a + ((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                            b + ((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4), dhi, idesc_s, kk > 0 ? 1u : 0u);
        };
        int n = 0, kt = 0;
        bool ok = true;
        for (int r = 0; ok && r < rounds; ++r) {
          const int item = pf_item_index(r, cl, nclusters);
          if (item >= p.num_items) continue;
          const PpItem it = pp_decode(p, item);
          if (!it.valid) continue;
          if (!(ok = wait_bounded(q_full, n & 1, abort_flag))) break;
          for (int t = 0; ok && t < it.n_kt; ++t) {
            const int g_t = kt + t;  // tile index over all items
            if (!(ok = wait_bounded(k_full, g_t & 1, abort_flag))) break;
#pragma unroll 1
            for (int i = 0; i < 2; ++i) {
              // slot i's score columns are free once its softmax read the previous tile
              if (g_t > 0 && !(ok = wait_bounded(&s_free[i], (g_t - 1) & 1, abort_flag))) break;
              tc_fence_after();
              issue_s(i);
              umma_commit_pair(&s_full[i], kBoth);
            }
            if (!ok) break;
            umma_commit_pair(k_empty, kBoth);
            if (t == it.n_kt - 1) umma_commit_pair(q_empty, kBoth);
          }
          kt += it.n_kt;
          ++n;
        }
      } else {
        constexpr uint32_t idesc_o = idesc_bf16_f32(256, 128, false, true);
        const uint32_t dP0 = desc_lo_sw128(sbase + kPpOffP, 16);
        const uint32_t dV0 = desc_lo_sw128(sbase + kPpOffV, 16384);  // MN-major, one 64-column atom per CTA
        // O_i += P_i V: 8 K-steps of 16 keys (A boxes 16 KB apart; B: 16 key rows = 2 KB)
        auto issue_pv = [&](int i, int vs, bool acc) {
          const uint32_t a = dP0 + static_cast<uint32_t>(i) * (kPpPBytes >> 4);
          const uint32_t d = tbase + 256 + static_cast<uint32_t>(i) * 128;
          const uint32_t bv = dV0 + static_cast<uint32_t>(vs) * (kPpVBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss_lo_pair(d, a + ((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                            bv + ((kk * 2048) >> 4), dhi, idesc_o, (acc || kk > 0) ? 1u : 0u);
        };
        int n = 0, kt = 0;
        bool ok = true;
        for (int r = 0; ok && r < rounds; ++r) {
          const int item = pf_item_index(r, cl, nclusters);
          if (item >= p.num_items) continue;
          const PpItem it = pp_decode(p, item);
          if (!it.valid) continue;
          for (int t = 0; ok && t < it.n_kt; ++t) {
            const int g_t = kt + t;
            if (!(ok = wait_bounded(&v_full[g_t & 1], (g_t >> 1) & 1, abort_flag))) break;
#pragma unroll 1
            for (int i = 0; i < 2; ++i) {
              if (!(ok = wait_bounded(&p_full[i], g_t & 1, abort_flag))) break;
              // an item's first P.V overwrites O: the previous item's epilogue must have read it
              if (t == 0 && n > 0 && !(ok = wait_bounded(&o_empty[i], (n - 1) & 1, abort_flag))) break;
              tc_fence_after();
              issue_pv(i, g_t & 1, t > 0);
              umma_commit_pair(&pv_done[i], kBoth);
            }
            if (!ok) break;
            umma_commit_pair(&v_empty[g_t & 1], kBoth);
          }
          kt += it.n_kt;
          ++n;
        }
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / epilogue (each CTA)
    setmaxnreg_inc<192>();
    const int i = warp >> 2;           // slot
    const int r = threadIdx.x & 127;   // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + i * 128;
    const uint32_t tO = tbase + lane_off + 256 + i * 128;
    const uint32_t sP = sbase + kPpOffP + i * kPpPBytes;
    const uint32_t b_sfree = lead(&s_free[i]), b_pfull = lead(&p_full[i]), b_oempty = lead(&o_empty[i]);
    int n = 0;   // items
    int kt = 0;  // key tiles over all items
    bool ok = true;
    for (int rr = 0; ok && rr < rounds; ++rr) {
      const int item = pf_item_index(rr, cl, nclusters);
      if (item >= p.num_items) continue;
      const PpItem it = pp_decode(p, item);
      if (!it.valid) continue;
      const int h = it.h0 + 2 * (int)rank + i;
      const int qpos = it.q0 + r;
      const float sg2 = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
      float m = sg2;
      float l = p.sinks ? 1.f : 0.f;   // exact row sum (lse)
      float lr = l;                    // sum of the bf16-rounded P that enter P.V (output)
      for (int t = 0; t < it.n_kt; ++t) {
        const int g_t = kt + t;
        const int kpos0 = (it.j_lo + t) * kPfTile;
        if (!(ok = wait_bounded(&s_full[i], g_t & 1, abort_flag))) break;
        tc_fence_after();
        float s[128];
        tmem_load128_sync(tS, s);
        tc_fence_before();
        __syncwarp();
        // S_i may now be overwritten by the next tile's scores (the loads are complete)
        if (lane == 0) mbar_arrive_cluster_relaxed(b_sfree);
        const bool full_tile = (kpos0 + kPfTile - 1 <= it.q0) &&
                               (p.window == 0 || (it.q0 + kPfTile - 1) - kpos0 <= p.window - 1);
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
        if (full_tile) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mx8[c & 7] = fmax3(mx8[c & 7], s[2 * c], s[2 * c + 1]);
        } else {
          const int hi_k = qpos - kpos0;
          const int lo_k = p.window > 0 ? qpos - p.window + 1 - kpos0 : -1;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            s[c] = (c <= hi_k && c >= lo_k) ? s[c] : -INFINITY;
            mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
          }
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_new = fmaxf(m, mx * p.scale_log2);
        float alpha = 1.f;
        bool rescale_o = false;
        if (m_new - m > kRescaleLog2) {  // false when both are -inf (NaN compare)
          alpha = ex2(m - m_new);
          l *= alpha;
          lr *= alpha;
          m = m_new;
          rescale_o = (t > 0);
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 acr[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float2 x = fma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
          const float2 e = make_float2(ex2(x.x), ex2(x.y));
          pk[c] = pack_bf16(e.x, e.y);
          acc[c & 1] = add2(acc[c & 1], e);
          acr[c & 1] = add2(acr[c & 1], make_float2(bf16_lo(pk[c]), bf16_hi(pk[c])));
        }
        const float2 a = add2(acc[0], acc[1]), ar = add2(acr[0], acr[1]);
        l += a.x + a.y;
        lr += ar.x + ar.y;
        // The P tile (and, when rescaling, O) are free once the previous P.V of this slot is done.
        if (g_t > 0 && !(ok = wait_bounded(&pv_done[i], (g_t - 1) & 1, abort_flag))) break;
        tc_fence_after();
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
          tmem_wait_st();
        }
        // P row r as bf16 into the K-major P tile: two boxes of [128 rows][64 keys],
        // 128-byte rows with the 16-byte chunk index XORed with row % 8
#pragma unroll
        for (int c16 = 0; c16 < 16; ++c16) {
          const uint32_t addr = sP + (c16 >> 3) * 16384 + r * 128 + ((((c16 & 7) ^ (r & 7))) << 4);
          st_shared_v4(addr, pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        // the leader's own P tile needs only CTA-scope ordering; the peer's, cluster scope
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(&p_full[i]);
          else
            mbar_arrive_cluster(b_pfull);
        }
      }
      if (!ok) break;
      // ---------------- epilogue: O / l -> out, lse (O read out of TMEM and released first)
      const int g_last = kt + it.n_kt - 1;
      kt += it.n_kt;
      if (!(ok = wait_bounded(&pv_done[i], g_last & 1, abort_flag))) break;
      tc_fence_after();
      float o[128];
      tmem_load128_sync(tO, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(b_oempty);  // O read (loads complete)
      ++n;
      if (qpos < it.len) {
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

  // Neither CTA leaves (or frees TMEM) while the other may still touch its
  // shared memory or TMEM: every MMA commit and remote arrival happens before this.
  tc_fence_before();
  cluster_sync();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace mimo
