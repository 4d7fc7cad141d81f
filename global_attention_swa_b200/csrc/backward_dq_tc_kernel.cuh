// Prefill backward, dQ on 5th-generation tensor cores (tcgen05).
//
// Gradient of the sliding-window / global attention with a learnable sink
// with respect to the queries (MiMo-V2-Flash model doc, "Key features":
// learnable attention-sink bias); the definitions are those of
// backward_kernel.cuh:
//   dq_i = s sum_j dS_ij k_j,   dS_ij = P_ij (v_scale <dO_i, v_j> - D_i),
//   P_ij = exp(s <q_i, k_j> - lse_i).
// Used when out and dout are bf16 (the fp32 form keeps the warp-level kernel).
//
// CTA = one 128-query tile of one query head (the 128 queries are the MMA
// rows and the TMEM lanes); it walks the 128-key tiles the tile sees.  Per
// key tile j:
//   S   = Q K^T     (SS, M=128 queries, N=128 keys, K=192)  -> TMEM, fp32
//   dP  = dO V^T    (SS, N=128 keys, K=128)                 -> TMEM, fp32
//   softmax warps:  P = 2^(S s log2e - lse log2e) (masked) in registers,
//                   dS = P (v_scale dP - D) rounded to bf16, written over dP
//   dQ += dS K      (TS: A = dS from TMEM, B = K MN-major, N=192, K=128 keys)
// and at the end writes dQ * s (fp32).
//
//   warps 0-3   softmax and epilogue, one query row (TMEM lane) per thread
//   warp 4      TMA producer (Q and dO once; K in two stages, V in one);
//               allocates / frees the 512 TMEM columns
//   warp 5      MMA issuer (one thread)
//
// TMEM columns: dQ [0,192)  S [192,320)  dP [320,448).  S(j+1) is issued as
// soon as the softmax has read S(j) into registers, so it overlaps the
// exponentials of tile j; dP(j+1) follows the dQ product of tile j, which
// consumes dS(j) from the dP columns.  Masking is a range of visible key
// columns per query row: one warp-uniform branch per tile, selects inside.
//
// Every wait is bounded (1 s of %globaltimer); a wait that gives up records
// MIMO_ERR_TIMEOUT and the CTA unwinds, freeing its TMEM.
#pragma once

#include "backward_kernel.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 9  // site numbers of the checked build

namespace mimo {

constexpr int kBdThreads = 192;
constexpr int kBdRows = 128;                         // queries per CTA
constexpr int kBdKeys = 128;                         // keys per tile
constexpr int kBdQBytes = kBdRows * 192 * 2;         // 3 boxes of [128 rows][64 dims]
constexpr int kBdOBytes = kBdRows * 128 * 2;         // 2 boxes (dO)
constexpr int kBdKBytes = kBdKeys * 192 * 2;         // 3 boxes
constexpr int kBdVBytes = kBdKeys * 128 * 2;         // 2 boxes
constexpr int kBdOffQ = 0;
constexpr int kBdOffO = kBdQBytes;                   // 49152
constexpr int kBdOffK = kBdOffO + kBdOBytes;         // 81920: 2 stages
constexpr int kBdOffV = kBdOffK + 2 * kBdKBytes;     // 180224
constexpr int kBdOffBar = kBdOffV + kBdVBytes;       // 212992
constexpr int kBdSmemBytes = kBdOffBar + 256 + 1024;
constexpr uint32_t kBdColDQ = 0, kBdColS = 192, kBdColDP = 320;

// P row of one key tile: P = 2^(S s log2e - lse log2e), zero outside the
// visible key columns [c_lo, c_hi] when kMasked (selects, no branches).
template <bool kMasked>
__device__ __forceinline__ void bwd_dq_p_row(float (&pr)[128], float scale_log2, float lse2,
                                             int c_lo, int c_hi) {
#pragma unroll
  for (int c = 0; c < 128; ++c) {
    const float x = ex2(fmaf(pr[c], scale_log2, -lse2));
    pr[c] = (!kMasked || (c >= c_lo && c <= c_hi)) ? x : 0.f;
  }
}

__global__ void __launch_bounds__(kBdThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t dqsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dqsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBdOffBar);
  uint64_t* qo_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* s_full = bars + 7;   // S(j) in TMEM
  uint64_t* s_free = bars + 8;   // S(j) read by the softmax
  uint64_t* dp_full = bars + 9;  // dP(j) in TMEM
  uint64_t* ds_full = bars + 10; // dS(j) written back
  uint64_t* done = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 13);
  uint64_t* mma_drain = bars + 14;  // teardown after a timed-out wait only
  volatile int* never_flag = reinterpret_cast<volatile int*>(bars + 15);  // never raised

  const int h = blockIdx.y, seq = blockIdx.z;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  if (!seq_in_bounds(b0, len, p.max_seqlen, p.total)) {  // bad cu_seqlens: touch nothing
    if (threadIdx.x == 0) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int nqt = (len + kBdRows - 1) / kBdRows;
  if ((int)blockIdx.x >= nqt) return;  // the whole CTA, before any barrier or TMEM
  const int qt = nqt - 1 - (int)blockIdx.x;  // the longest key loops are issued first
  const int q0 = qt * kBdRows;
  const int g = h / p.G;
  const int last_q = min(q0 + kBdRows - 1, len - 1);
  const int kt_lo = p.window > 0 ? max(0, q0 - p.window + 1) / kBdKeys : 0;
  const int n_kt = last_q / kBdKeys - kt_lo + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int armed_qo = 0, armed_k = 0, armed_v = 0;  // phases the producer armed (K: tiles in order)
  if (warp == 4) {
    if (lane == 0) {
      mbar_init(qo_full, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&k_full[i], 1);
        mbar_init(&k_empty[i], 1);
      }
      mbar_init(v_full, 1);
      mbar_init(v_empty, 1);
      mbar_init(s_full, 1);
      mbar_init(s_free, 128);
      mbar_init(mma_drain, 1);
      *never_flag = 0;
      mbar_init(dp_full, 1);
      mbar_init(ds_full, 128);
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
  const int nt = *abort_flag ? 0 : n_kt;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(qo_full, kBdQBytes + kBdOBytes);
      ++armed_qo;
#pragma unroll
      for (int c = 0; c < 3; ++c) tma_load_3d(smem + kBdOffQ + c * 16384, &tm_q, qo_full, c * 64, h, b0 + q0);
#pragma unroll
      for (int c = 0; c < 2; ++c) tma_load_3d(smem + kBdOffO + c * 16384, &tm_do, qo_full, c * 64, h, b0 + q0);
      for (int t = 0; t < nt; ++t) {
        const int ks = t & 1;
        const int row = b0 + (kt_lo + t) * kBdKeys;
        if (t >= 2 && !wait_bounded(&k_empty[ks], ((t >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[ks], kBdKBytes);
        ++armed_k;
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_3d(smem + kBdOffK + ks * kBdKBytes + c * 16384, &tm_k, &k_full[ks], c * 64, g, row);
        if (t >= 1 && !wait_bounded(v_empty, (t - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(v_full, kBdVBytes);
        ++armed_v;
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_3d(smem + kBdOffV + c * 16384, &tm_v, v_full, c * 64, g, row);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nt > 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_q = idesc_bf16_f32(128, 192, false, true);
      constexpr uint32_t dhi = desc_hi_sw128(1024);
      const uint32_t dQ = desc_lo_sw128(sbase + kBdOffQ, 16);
      const uint32_t dO = desc_lo_sw128(sbase + kBdOffO, 16);
      const uint32_t dK0 = desc_lo_sw128(sbase + kBdOffK, 16);       // K-major (scores)
      const uint32_t dKm0 = desc_lo_sw128(sbase + kBdOffK, 16384);   // MN-major (dQ product)
      const uint32_t dV = desc_lo_sw128(sbase + kBdOffV, 16);
      constexpr uint32_t kKStep = kBdKBytes >> 4;
      const uint32_t tDQ = tbase + kBdColDQ, tS = tbase + kBdColS, tDP = tbase + kBdColDP;
      // S = Q K^T: 12 K-steps of 16 dims (3 swizzle boxes x 4 steps of 32 B)
      auto issue_s = [&](int ks) {
        const uint32_t b = dK0 + ks * kKStep;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss_lo(tS, dQ + off, b + off, dhi, id_s, kk > 0 ? 1u : 0u);
        }
      };
      // dP = dO V^T: 8 K-steps
      auto issue_dp = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss_lo(tDP, dO + off, dV + off, dhi, id_s, kk > 0 ? 1u : 0u);
        }
      };
      // dQ += dS K: 8 K-steps of 16 keys (A: 8 TMEM columns; B: 16 key rows = 2 KB)
      auto issue_dq = [&](int j) {
        const uint32_t b = dKm0 + (j & 1) * kKStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts_lo(tDQ, tDP + kk * 8, b + ((kk * 2048) >> 4), dhi, id_q, (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bounded(qo_full, 0, abort_flag) && wait_bounded(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        umma_commit(s_full);
      }
      if (ok && (ok = wait_bounded(v_full, 0, abort_flag))) {
        tc_fence_after();
        issue_dp();
        umma_commit(dp_full);
        umma_commit(v_empty);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const bool more = j + 1 < nt;
        if (more) {
          // S(j+1) once the softmax holds S(j) in registers
          if (!(ok = wait_bounded(s_free, j & 1, abort_flag))) break;
          if (!(ok = wait_bounded(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s((j + 1) & 1);
          umma_commit(s_full);
        }
        if (!(ok = wait_bounded(ds_full, j & 1, abort_flag))) break;
        tc_fence_after();
        issue_dq(j);
        umma_commit(&k_empty[j & 1]);
        if (more) {
          if (!(ok = wait_bounded(v_full, (j + 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_dp();
          umma_commit(dp_full);
          umma_commit(v_empty);
        }
      }
      if (ok) umma_commit(done);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = threadIdx.x;  // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int q = q0 + r;
    const bool live = q < len && MIMO_ROW_OK((long long)(b0 + q) * p.Hq + h, (long long)p.total * p.Hq);
    const size_t li = (size_t)h * p.total + b0 + q;
    const float lse2 = live ? p.lse[li] * 1.4426950408889634f : 0.f;
    const float Dq = live ? p.D[li] : 0.f;
    bool ok = nt > 0;
    for (int j = 0; ok && j < nt; ++j) {
      const int k0 = (kt_lo + j) * kBdKeys;
      // visible key columns of this query row: [c_lo, c_hi] (empty when c_hi < c_lo)
      const int c_lo = p.window > 0 ? max(q - p.window + 1 - k0, 0) : 0;
      const int c_hi = live ? min(min(q, len - 1) - k0, kBdKeys - 1) : -1;
      const bool full = __all_sync(0xffffffffu, c_lo == 0 && c_hi == kBdKeys - 1);
      if (!(ok = wait_bounded(s_full, j & 1, abort_flag))) break;
      tc_fence_after();
      float pr[128];
      tmem_load128_sync(tbase + lane_off + kBdColS, pr);
      tc_fence_before();
      mbar_arrive(s_free);  // the S columns may be overwritten by S(j+1)
      if (full)
        bwd_dq_p_row<false>(pr, p.scale_log2, lse2, c_lo, c_hi);
      else
        bwd_dq_p_row<true>(pr, p.scale_log2, lse2, c_lo, c_hi);
      if (!(ok = wait_bounded(dp_full, j & 1, abort_flag))) break;
      tc_fence_after();
      // dS = P (v_scale dP - D) in four chunks of 32 keys; chunk c lands in the
      // (already read) columns [16 c, 16 c + 16) of the dP buffer as bf16 pairs
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float dp[32];
        tmem_load32_sync(tbase + lane_off + kBdColDP + 32 * c, dp);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float d0 = pr[32 * c + 2 * e] * fmaf(p.v_scale, dp[2 * e], -Dq);
          const float d1 = pr[32 * c + 2 * e + 1] * fmaf(p.v_scale, dp[2 * e + 1], -Dq);
          pk[e] = pack_bf16(d0, d1);
        }
        tmem_st16(tbase + lane_off + kBdColDP + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ---------------- epilogue: dQ * scale for the tile's valid rows
    if (ok && wait_bounded(done, 0, abort_flag)) {
      tc_fence_after();
      float* dqr = p.dq + ((size_t)(b0 + q) * p.Hq + h) * kBwQK;
#pragma unroll 1
      for (int c = 0; c < 6; ++c) {
        float o[32];
        tmem_load32_sync(tbase + lane_off + kBdColDQ + 32 * c, o);
        if (live) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dqr + 32 * c)[e] =
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
      drain_armed(qo_full, armed_qo, never_flag);
      drain_armed(&k_full[0], (armed_k + 1) / 2, never_flag);
      drain_armed(&k_full[1], armed_k / 2, never_flag);
      drain_armed(v_full, armed_v, never_flag);
    }
    if (warp == 5 && lane == 0 && nt > 0) drain_mma(mma_drain, never_flag);  // nt > 0: MMAs may have been issued
    __syncthreads();
  }
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace mimo
