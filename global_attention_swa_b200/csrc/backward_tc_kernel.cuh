// Prefill backward, dK and dV on 5th-generation tensor cores (tcgen05).
//
// Gradients of the sliding-window / global attention with a learnable sink
// (MiMo-V2-Flash model doc, "Key features"); the definitions are those of
// backward_kernel.cuh.  This kernel replaces the two warp-level dV / dK
// passes when out and dout are bf16.
//
// CTA = one 128-key tile of one key/value head (the 128 keys are the MMA rows
// and the TMEM lanes).  It walks the items (query head of the group, 64-query
// tile that sees the keys); per item:
//   S^T  = K Q^T     (SS, M=128 keys, N=64 queries, K=192)  -> TMEM, fp32
//   dP^T = V dO^T    (SS, N=64, K=128)                       -> TMEM, fp32
//   softmax warps:   P^T = 2^(S^T s log2e - lse log2e) (masked),
//                    dS^T = P^T (v_scale dP^T - D), both rounded to bf16 and
//                    written over their fp32 sources
//   dV += P^T dO     (TS: A = P^T from TMEM, B = dO MN-major, N=128, K=64)
//   dK += dS^T Q     (TS: A = dS^T from TMEM, B = Q MN-major,  N=192, K=64)
// and at the end writes dV * v_scale and dK * scale (fp32).
//
//   warps 0-3   softmax and epilogue, one key row (TMEM lane) per thread
//   warp 4      TMA producer (K, V once; Q and dO per item, three stages);
//               allocates / frees the 512 TMEM columns
//   warp 5      MMA issuer (one thread)
//
// TMEM columns: dV [0,128)  dK [128,320)  S^T_0 [320,384)  dP^T [384,448)
// S^T_1 [448,512).  The next item's S^T goes to the other buffer while the
// softmax works on the current one; its dP^T follows the current dK product.
// The softmax hands its results over in two steps: P^T (the dV product can
// start) and then dS^T (the dK product), so the exponentials of one item
// overlap the dK and next dP^T products of the item before.  Masking is per
// key row as a range of visible query columns: one warp-uniform branch per
// item (all visible / some masked), selects inside.
//
// Every wait is bounded (1 s of %globaltimer); a wait that gives up records
// MIMO_ERR_TIMEOUT and the CTA unwinds, freeing its TMEM.
#pragma once

#include "backward_kernel.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 8  // site numbers of the checked build

namespace mimo {

constexpr int kBtThreads = 192;
constexpr int kBtKeys = 128;                  // key rows per CTA
constexpr int kBtQ = 64;                      // queries per item
constexpr int kBtKBytes = 128 * 192 * 2;      // 3 boxes of [128 keys][64 dims]
constexpr int kBtVBytes = 128 * 128 * 2;      // 2 boxes
constexpr int kBtQBytes = 64 * 192 * 2;       // 3 boxes of [64 queries][64 dims]
constexpr int kBtOBytes = 64 * 128 * 2;       // 2 boxes (dO)
constexpr int kBtStage = kBtQBytes + kBtOBytes;
constexpr int kBtOffK = 0;
constexpr int kBtOffV = kBtKBytes;
constexpr int kBtStages = 3;
constexpr int kBtOffStage = kBtOffV + kBtVBytes;
constexpr int kBtOffLD = kBtOffStage + kBtStages * kBtStage;  // 2 x {lse log2e [64], D [64]}
constexpr int kBtOffBar = kBtOffLD + 2 * 2 * kBtQ * 4;
constexpr int kBtSmemBytes = kBtOffBar + 256 + 1024;      // barriers + alignment slack
constexpr uint32_t kBtColDV = 0, kBtColDK = 128, kBtColS0 = 320, kBtColDP = 384, kBtColS1 = 448;

// P^T row of one item: P = 2^(S s log2e - lse log2e) for the 64 query columns
// (lse log2e in ld4[0..15]), zero outside [c_lo, c_hi] when kMasked (selects,
// no branches); also packed to bf16 pairs for the dV product.
template <bool kMasked>
__device__ __forceinline__ void bwd_p_tile(float (&pe)[64], const float4* ld4, float scale_log2,
                                           int c_lo, int c_hi, uint32_t (&pk)[32]) {
#pragma unroll
  for (int c4 = 0; c4 < 16; ++c4) {
    const float4 l4 = ld4[c4];
    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int qc = 4 * c4 + e;
      const float x = ex2(fmaf(pe[qc], scale_log2, -lv[e]));
      pe[qc] = (!kMasked || (qc >= c_lo && qc <= c_hi)) ? x : 0.f;
    }
    pk[2 * c4] = pack_bf16(pe[4 * c4], pe[4 * c4 + 1]);
    pk[2 * c4 + 1] = pack_bf16(pe[4 * c4 + 2], pe[4 * c4 + 3]);
  }
}

__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t tsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBtOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;   // [kBtStages]
  uint64_t* q_empty = bars + 4;  // [kBtStages]
  uint64_t* s_full = bars + 7;    // [2] S^T of items with j & 1 == b is in TMEM
  uint64_t* p_full = bars + 9;    // [2] P^T of those items written back (bf16)
  uint64_t* dp_full = bars + 11;  // dP^T of the current item is in TMEM
  uint64_t* ds_full = bars + 12;  // dS^T of the current item written back (bf16)
  uint64_t* ld_full = bars + 13;  // [2]
  uint64_t* done = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 17);
  uint64_t* mma_drain = bars + 18;  // teardown after a timed-out wait only
  volatile int* never_flag = reinterpret_cast<volatile int*>(bars + 19);  // never raised
  float* sLD = reinterpret_cast<float*>(smem + kBtOffLD);

  // key tiles in ascending order, KV heads fastest: the longest causal loops start first
  const int kt = (int)blockIdx.x / p.Hkv, g = (int)blockIdx.x % p.Hkv, seq = blockIdx.y;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  if (!seq_in_bounds(b0, len, p.max_seqlen, p.total)) {  // bad cu_seqlens: touch nothing
    if (threadIdx.x == 0) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int k0 = kt * kBtKeys;
  if (k0 >= len) return;  // the whole CTA, before any barrier or TMEM
  const int kv = min(kBtKeys, len - k0);
  const int last_k = k0 + kv - 1;
  const int qt_lo = k0 / kBtQ;
  const int qt_hi = p.window > 0 ? min((len - 1) / kBtQ, (last_k + p.window - 1) / kBtQ) : (len - 1) / kBtQ;
  const int nq = qt_hi - qt_lo + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int armed_kv = 0, armed_q = 0;  // phases the producer armed: K/V once, Q/dO per item (stage j % 3)
  if (warp == 4) {
    if (lane == 0) {
      mbar_init(kv_full, 1);
      for (int i = 0; i < kBtStages; ++i) {
        mbar_init(&q_full[i], 1);
        mbar_init(&q_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&ld_full[i], 128);
        mbar_init(&s_full[i], 1);
        mbar_init(&p_full[i], 128);
      }
      mbar_init(dp_full, 1);
      mbar_init(ds_full, 128);
      mbar_init(mma_drain, 1);
      *never_flag = 0;
      mbar_init(done, 1);
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
  const int items = *abort_flag ? 0 : p.G * nq;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && items > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, kBtKBytes + kBtVBytes);
      ++armed_kv;
#pragma unroll
      for (int c = 0; c < 3; ++c) tma_load_3d(smem + kBtOffK + c * 16384, &tm_k, kv_full, c * 64, g, b0 + k0);
#pragma unroll
      for (int c = 0; c < 2; ++c) tma_load_3d(smem + kBtOffV + c * 16384, &tm_v, kv_full, c * 64, g, b0 + k0);
      for (int j = 0; j < items; ++j) {
        const int st = j % kBtStages;
        if (j >= kBtStages && !wait_bounded(&q_empty[st], (j / kBtStages - 1) & 1, abort_flag)) break;
        const int h = g * p.G + j / nq;
        const int row = b0 + (qt_lo + j % nq) * kBtQ;
        uint8_t* stg = smem + kBtOffStage + st * kBtStage;
        mbar_arrive_expect_tx(&q_full[st], kBtStage);
        ++armed_q;
#pragma unroll
        for (int c = 0; c < 3; ++c) tma_load_3d(stg + c * 8192, &tm_q, &q_full[st], c * 64, h, row);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_3d(stg + kBtQBytes + c * 8192, &tm_do, &q_full[st], c * 64, h, row);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && items > 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_v = idesc_bf16_f32(128, 128, false, true);
      constexpr uint32_t id_k = idesc_bf16_f32(128, 192, false, true);
      constexpr uint32_t dhi = desc_hi_sw128(1024);
      const uint32_t dK = desc_lo_sw128(sbase + kBtOffK, 16);
      const uint32_t dV = desc_lo_sw128(sbase + kBtOffV, 16);
      // Q / dO stages: K-major B for the score products; MN-major B (64-dim
      // atoms one 8 KB box apart) for the accumulations over queries
      const uint32_t dQk0 = desc_lo_sw128(sbase + kBtOffStage, 16);
      const uint32_t dOk0 = desc_lo_sw128(sbase + kBtOffStage + kBtQBytes, 16);
      const uint32_t dQm0 = desc_lo_sw128(sbase + kBtOffStage, 8192);
      const uint32_t dOm0 = desc_lo_sw128(sbase + kBtOffStage + kBtQBytes, 8192);
      constexpr uint32_t kStageStep = kBtStage >> 4;
      const uint32_t tDV = tbase + kBtColDV, tDK = tbase + kBtColDK, tDP = tbase + kBtColDP;
      auto tS = [&](int j) { return tbase + ((j & 1) ? kBtColS1 : kBtColS0); };
      // S^T = K Q^T: 12 K-steps of 16 dims (A boxes 16 KB apart, B boxes 8 KB apart)
      auto issue_s = [&](uint32_t t, int st) {
        const uint32_t b = dQk0 + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk)
          umma_ss_lo(t, dK + ((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                     b + ((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4), dhi, id_s, kk > 0 ? 1u : 0u);
      };
      // dP^T = V dO^T: 8 K-steps
      auto issue_dp = [&](int st) {
        const uint32_t b = dOk0 + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss_lo(tDP, dV + ((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                     b + ((((kk >> 2) * 8192) + (kk & 3) * 32) >> 4), dhi, id_s, kk > 0 ? 1u : 0u);
      };
      // dV += P^T dO and dK += dS^T Q: 4 K-steps of 16 queries each (A: 8 TMEM
      // columns; B: 16 rows = 2 KB)
      auto issue_dv = [&](int j, int st) {
        const uint32_t tP = tS(j), bo = dOm0 + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts_lo(tDV, tP + kk * 8, bo + ((kk * 2048) >> 4), dhi, id_v, (j > 0 || kk > 0) ? 1u : 0u);
      };
      auto issue_dk = [&](int j, int st) {
        const uint32_t bq = dQm0 + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts_lo(tDK, tDP + kk * 8, bq + ((kk * 2048) >> 4), dhi, id_k, (j > 0 || kk > 0) ? 1u : 0u);
      };
      // Per item j the softmax hands over P^T first (-> dV) and dS^T second
      // (-> dK); the next item's S^T is issued one item ahead into the other
      // buffer, its dP^T once dK has consumed the dP buffer.
      bool ok = wait_bounded(kv_full, 0, abort_flag) && wait_bounded(&q_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(tS(0), 0);
        umma_commit(&s_full[0]);
        issue_dp(0);
        umma_commit(dp_full);
      }
      for (int j = 0; ok && j < items; ++j) {
        const int st = j % kBtStages;
        const int sn = (j + 1) % kBtStages;
        const bool more = j + 1 < items;
        if (more) {
          if (!(ok = wait_bounded(&q_full[sn], ((j + 1) / kBtStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(tS(j + 1), sn);  // overlaps the softmax of item j
          umma_commit(&s_full[(j + 1) & 1]);
        }
        if (!(ok = wait_bounded(&p_full[j & 1], (j >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        issue_dv(j, st);
        if (!(ok = wait_bounded(ds_full, j & 1, abort_flag))) break;
        tc_fence_after();
        issue_dk(j, st);
        umma_commit(&q_empty[st]);
        if (more) {
          issue_dp(sn);
          umma_commit(dp_full);
        }
      }
      if (ok) umma_commit(done);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = threadIdx.x;  // TMEM lane == key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int key = k0 + r;
    // one value per thread of each item's lse (base 2, threads 0-63) or D
    // (threads 64-127), loaded one item ahead and passed on through shared memory
    auto fetch = [&](int j) -> float {
      const int qp = (qt_lo + j % nq) * kBtQ + (r & (kBtQ - 1));
      if (qp >= len) return 0.f;
      const size_t gi = (size_t)(g * p.G + j / nq) * p.total + b0 + qp;
      if (!MIMO_ROW_OK(gi, (long long)p.Hq * p.total)) return 0.f;
      return r < kBtQ ? p.lse[gi] * 1.4426950408889634f : p.D[gi];
    };
    bool ok = items > 0;
    float nxt = ok ? fetch(0) : 0.f;
    for (int j = 0; ok && j < items; ++j) {
      const int q0 = (qt_lo + j % nq) * kBtQ;
      float* ld = sLD + (j & 1) * 2 * kBtQ;
      ld[r] = nxt;
      mbar_arrive(&ld_full[j & 1]);
      if (j + 1 < items) nxt = fetch(j + 1);  // in flight during this item
      if (!(ok = wait_bounded(&ld_full[j & 1], (j >> 1) & 1, abort_flag))) break;
      // visible query columns of this key row: [c_lo, c_hi] (empty when c_hi < c_lo)
      const int c_lo = max(key - q0, 0);
      int c_hi = min(len - 1 - q0, kBtQ - 1);
      if (p.window > 0) c_hi = min(c_hi, key + p.window - 1 - q0);
      if (key >= len) c_hi = -1;
      // one branch per warp and item: every row sees every query, or selects per element
      const bool full = __all_sync(0xffffffffu, c_lo == 0 && c_hi == kBtQ - 1);
      // ---- P^T = 2^(S^T s log2e - lse log2e), rounded to bf16 over S^T -> dV
      if (!(ok = wait_bounded(&s_full[j & 1], (j >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t tSr = tbase + lane_off + ((j & 1) ? kBtColS1 : kBtColS0);
      const uint32_t tDPr = tbase + lane_off + kBtColDP;
      const float4* ld4 = reinterpret_cast<const float4*>(ld);  // [0,16): lse log2e, [16,32): D
      float pe[64];
      tmem_load64_sync(tSr, pe);
      {
        uint32_t pk[32];
        if (full)
          bwd_p_tile<false>(pe, ld4, p.scale_log2, c_lo, c_hi, pk);
        else
          bwd_p_tile<true>(pe, ld4, p.scale_log2, c_lo, c_hi, pk);
        tmem_st32(tSr, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
      // ---- dS^T = P^T (v_scale dP^T - D), rounded to bf16 over dP^T -> dK
      if (!(ok = wait_bounded(dp_full, j & 1, abort_flag))) break;
      tc_fence_after();
      {
        float dp[64];
        tmem_load64_sync(tDPr, dp);
        uint32_t dk[32];
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 d4 = ld4[16 + c4];
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
          float de[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) de[e] = pe[4 * c4 + e] * fmaf(p.v_scale, dp[4 * c4 + e], -dv4[e]);
          dk[2 * c4] = pack_bf16(de[0], de[1]);
          dk[2 * c4 + 1] = pack_bf16(de[2], de[3]);
        }
        tmem_st32(tDPr, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ---------------- epilogue: dV * v_scale and dK * scale for valid keys
    if (ok && wait_bounded(done, 0, abort_flag)) {
      tc_fence_after();
      const bool valid = r < kv && MIMO_ROW_OK((long long)(b0 + key) * p.Hkv + g, (long long)p.total * p.Hkv);
      float* dvr = p.dv + ((size_t)(b0 + key) * p.Hkv + g) * kBwV;
      float* dkr = p.dk + ((size_t)(b0 + key) * p.Hkv + g) * kBwQK;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_load32_sync(tbase + lane_off + kBtColDV + 32 * c, o);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dvr + 32 * c)[e] =
                make_float4(o[4 * e] * p.v_scale, o[4 * e + 1] * p.v_scale, o[4 * e + 2] * p.v_scale,
                            o[4 * e + 3] * p.v_scale);
        }
      }
#pragma unroll 1
      for (int c = 0; c < 6; ++c) {
        float o[32];
        tmem_load32_sync(tbase + lane_off + kBtColDK + 32 * c, o);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dkr + 32 * c)[e] =
                make_float4(o[4 * e] * p.scale, o[4 * e + 1] * p.scale, o[4 * e + 2] * p.scale,
                            o[4 * e + 3] * p.scale);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // a role gave up: the loads and MMAs still in flight land before the CTA
    // frees its TMEM and exits
    if (warp == 4 && lane == 0) {
      drain_armed(kv_full, armed_kv, never_flag);
      for (int s = 0; s < kBtStages; ++s)
        drain_armed(&q_full[s], armed_q > s ? (armed_q - 1 - s) / kBtStages + 1 : 0, never_flag);
    }
    if (warp == 5 && lane == 0 && items > 0) drain_mma(mma_drain, never_flag);  // items > 0: MMAs may have been issued
    __syncthreads();
  }
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace mimo
