// Prefill: packed variable-length causal GQA attention with a sliding window
// and a per-head attention sink, on 5th-generation tensor cores (tcgen05).
//
// MiMo-V2-Flash model doc, "Key features" (hybrid attention: 5:1 sliding
// window / global layers, small window, learnable attention-sink bias) and
// MiMoV2FlashConfig (64 query heads over 4 key/value heads, head_dim 192 for
// query/key, v_head_dim 128, sliding_window 129).
//
// One CTA = one 128-query tile of one sequence x two query heads of the same
// key/value group.  Both heads see exactly the same key tiles, so each K/V
// tile staged in shared memory feeds two 128x128 score tiles.
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
// warpgroup gives back down to 80 and the two softmax warpgroups take 208
// (2*128*208 + 128*80 = 63488 <= 384*168 = 64512; per SM sub-partition
// 208 + 208 + 80 registers x 32 lanes = 15872 <= 16384).
//
// TMEM columns: S_0 [0,128)  S_1 [128,256)  O_0 [256,384)  O_1 [384,512).
// P_i (bf16, two per 32-bit column) overwrites the first 64 columns of S_i.
//
// Online softmax in base 2 with the sink folded into the running state:
// m starts at sigma_h*log2(e) and l at 1 (the sink's own term), so the sink
// enters the normaliser once and never the output.  The running max is only
// moved (and O rescaled) when a row's max grows by more than kRescaleLog2;
// otherwise P is computed against the stale max (P <= 2^kRescaleLog2), which
// is exact because O and l share the same reference.
//
// Key tiles wholly outside [q0 - window + 1, q0 + 127] are never loaded: a
// 129-wide window touches at most two 128-key tiles per query tile.
#pragma once

#include "common.cuh"

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
constexpr float kRescaleLog2 = 8.0f;

struct PrefillParams {
  const int32_t* cu_seqlens;  // [num_seqs + 1]
  const float* sinks;         // [Hq] or null
  void* out;                  // [total, Hq, 128]
  float* lse;                 // [Hq, total] or null
  int total, Hq, Hkv, G;
  int window;
  int pairs_per_group;        // ceil(G / 2)
  float scale_log2;           // softmax_scale * log2(e)
  float v_scale;
  int out_f32;
};

// K-major operand (rows of 64 bf16 = 128 B, 8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  return smem_desc_sw128(addr, 16, 1024);
}
// MN-major operand V: 64-column atoms 16 KB apart (LBO), 8-key groups 1024 B apart (SBO).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr) {
  return smem_desc_sw128(addr, 16384, 1024);
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t psmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(psmem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPfOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* s_full = bars + 7;   // [2]
  uint64_t* p_full = bars + 9;   // [2]
  uint64_t* o_full = bars + 11;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = blockIdx.z;
  const int b0 = p.cu_seqlens[seq];
  const int len = p.cu_seqlens[seq + 1] - b0;
  const int qt = gridDim.x - 1 - blockIdx.x;  // longest (last) tiles first
  const int q0 = qt * kPfTile;
  if (q0 >= len || timed_out_before()) return;
  const int g = blockIdx.y / p.pairs_per_group;
  const int pp = blockIdx.y % p.pairs_per_group;
  const int h0 = g * p.G + 2 * pp;
  const bool has1 = (2 * pp + 1) < p.G;
  const int h1 = h0 + 1;

  const int last_q = min(q0 + kPfTile - 1, len - 1);
  const int j_hi = last_q / kPfTile;
  const int j_lo = p.window > 0 ? max(0, q0 - p.window + 1) / kPfTile : 0;
  const int n_kt = j_hi - j_lo + 1;

  if (warp == 8) {
    if (lane == 0) {
      mbar_init(q_full, 1);
      mbar_init(&k_full[0], 1);
      mbar_init(&k_full[1], 1);
      mbar_init(&k_empty[0], 1);
      mbar_init(&k_empty[1], 1);
      mbar_init(v_full, 1);
      mbar_init(v_empty, 1);
      mbar_init(&s_full[0], 1);
      mbar_init(&s_full[1], 1);
      mbar_init(&p_full[0], 128);
      mbar_init(&p_full[1], 128);
      mbar_init(&o_full[0], 1);
      mbar_init(&o_full[1], 1);
      *abort_flag = 0;
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
  if (warp >= 8) {
    setmaxnreg_dec<80>();
  }
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, has1 ? 2 * kPfQBytes : kPfQBytes);
#pragma unroll
      for (int c = 0; c < 3; ++c)
        tma_load_3d(smem + kPfOffQ0 + c * 16384, &tm_q, q_full, c * 64, h0, b0 + q0);
      if (has1) {
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_3d(smem + kPfOffQ1 + c * 16384, &tm_q, q_full, c * 64, h1, b0 + q0);
      }
      for (int t = 0; t < n_kt; ++t) {
        const int row = b0 + (j_lo + t) * kPfTile;
        const int ks = t & 1;
        if (t >= 2 && !wait_bounded(&k_empty[ks], ((t >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[ks], kPfKBytes);
#pragma unroll
        for (int c = 0; c < 3; ++c)
          tma_load_3d(smem + kPfOffK + ks * kPfKBytes + c * 16384, &tm_k, &k_full[ks], c * 64, g, row);
        if (t >= 1 && !wait_bounded(v_empty, (t - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(v_full, kPfVBytes);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + kPfOffV + c * 16384, &tm_v, v_full, c * 64, g, row);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      const uint32_t tS0 = tbase + 0, tS1 = tbase + 128, tO0 = tbase + 256, tO1 = tbase + 384;
      const uint32_t aQ0 = sbase + kPfOffQ0, aQ1 = sbase + kPfOffQ1;
      bool ok = wait_bounded(q_full, 0, abort_flag);
      // S_i = Q_i K^T over 192 dims = 12 MMAs of K=16 (3 swizzle boxes x 4 steps of 32 B)
      auto issue_s = [&](uint32_t tS, uint32_t aQ, uint32_t aK) {
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, kmajor_desc(aQ + off), kmajor_desc(aK + off), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_i += P_i V over 128 keys = 8 MMAs of K=16 (P: 8 TMEM columns each; V: 16 rows = 2 KB)
      auto issue_pv = [&](uint32_t tO, uint32_t tP, bool acc) {
        const uint32_t aV = sbase + kPfOffV;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tO, tP + kk * 8, mnmajor_desc(aV + kk * 2048), idesc_o, (acc || kk > 0) ? 1u : 0u);
      };
      if (ok) ok = wait_bounded(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        const uint32_t aK = sbase + kPfOffK;
        issue_s(tS0, aQ0, aK);
        umma_commit(&s_full[0]);
        if (has1) {
          issue_s(tS1, aQ1, aK);
          umma_commit(&s_full[1]);
        }
        umma_commit(&k_empty[0]);
      }
      for (int t = 0; ok && t < n_kt; ++t) {
        const bool last = (t == n_kt - 1);
        if (!wait_bounded(v_full, t & 1, abort_flag)) break;
        if (!wait_bounded(&p_full[0], t & 1, abort_flag)) break;
        tc_fence_after();
        issue_pv(tO0, tS0, t > 0);
        if (last) umma_commit(&o_full[0]);
        const int kn = (t + 1) & 1;
        if (!last) {
          if (!wait_bounded(&k_full[kn], ((t + 1) >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          issue_s(tS0, aQ0, sbase + kPfOffK + kn * kPfKBytes);
          umma_commit(&s_full[0]);
        }
        if (has1) {
          if (!wait_bounded(&p_full[1], t & 1, abort_flag)) break;
          tc_fence_after();
          issue_pv(tO1, tS1, t > 0);
          if (last) umma_commit(&o_full[1]);
        }
        umma_commit(v_empty);
        if (!last) {
          if (has1) {
            issue_s(tS1, aQ1, sbase + kPfOffK + kn * kPfKBytes);
            umma_commit(&s_full[1]);
          }
          umma_commit(&k_empty[kn]);
        }
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / epilogue
    setmaxnreg_inc<208>();
    const int i = warp >> 2;  // which head of the pair
    if (i == 0 || has1) {
      const int h = i ? h1 : h0;
      const int r = threadIdx.x & 127;  // TMEM lane == query row within the tile
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t tS = tbase + lane_off + i * 128;
      const uint32_t tO = tbase + lane_off + 256 + i * 128;
      const int qpos = q0 + r;
      const float sg2 = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
      float m = sg2;
      float l = p.sinks ? 1.f : 0.f;
      bool ok = true;
      for (int t = 0; t < n_kt; ++t) {
        const int kpos0 = (j_lo + t) * kPfTile;
        if (!wait_bounded(&s_full[i], t & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32f(tS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_wait_ld();
        const bool full_tile = (kpos0 + kPfTile - 1 <= q0) &&
                               (p.window == 0 || (q0 + kPfTile - 1) - kpos0 <= p.window - 1);
        // Row max of the raw scores (the scale is positive, so it commutes with
        // max), as 8 independent chains to keep the dependency depth short.
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
        if (full_tile) {
#pragma unroll
          for (int c = 0; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
        } else {
          const int hi_k = qpos - kpos0;                                  // keys <= hi_k visible
          const int lo_k = p.window > 0 ? qpos - p.window + 1 - kpos0 : -1;  // keys >= lo_k visible
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            s[c] = (c <= hi_k && c >= lo_k) ? s[c] : -INFINITY;
            mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
          }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_new = fmaxf(m, mx * p.scale_log2);
        float alpha = 1.f;
        bool rescale_o = false;
        if (m_new - m > kRescaleLog2) {  // false when both are -inf (NaN compare)
          alpha = ex2(m - m_new);
          l *= alpha;
          m = m_new;
          rescale_o = (t > 0);
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        // P = 2^(s*scale - m), rounded to bf16 for the PV product; the row sum
        // keeps the unrounded values so that lse stays exact to fp32.
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 x = fma2(make_float2(s[64 * half + 2 * c], s[64 * half + 2 * c + 1]), sc2, nm2);
            const float2 e = make_float2(ex2(x.x), ex2(x.y));
            pk[c] = pack_bf16(e.x, e.y);
            acc[c & 3] = add2(acc[c & 3], e);
          }
          tmem_st32(tS + 32 * half, pk);
        }
        const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
        const float2 a = add2(a01, a23);
        const float rs = a.x + a.y;
        l += rs;
        // O of the previous tile is complete here: S_i(t) was committed after PV_i(t-1).
        if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
            const float a = rescale_o ? alpha : 1.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[i]);
      }
      // ---------------- epilogue: O / l -> out, lse
      if (ok && wait_bounded(&o_full[i], 0, abort_flag)) {
        tc_fence_after();
        const bool valid = qpos < len;
        const int tok = b0 + qpos;
        const float f = (l > 0.f) ? p.v_scale / l : 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          if (valid) {
            const size_t ob = ((size_t)tok * p.Hq + h) * 128 + c * 32;
            if (p.out_f32) {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + ob);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * f, __uint_as_float(o[4 * e + 1]) * f,
                                     __uint_as_float(o[4 * e + 2]) * f, __uint_as_float(o[4 * e + 3]) * f);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 u;
                u.x = pack_bf16(__uint_as_float(o[8 * e + 0]) * f, __uint_as_float(o[8 * e + 1]) * f);
                u.y = pack_bf16(__uint_as_float(o[8 * e + 2]) * f, __uint_as_float(o[8 * e + 3]) * f);
                u.z = pack_bf16(__uint_as_float(o[8 * e + 4]) * f, __uint_as_float(o[8 * e + 5]) * f);
                u.w = pack_bf16(__uint_as_float(o[8 * e + 6]) * f, __uint_as_float(o[8 * e + 7]) * f);
                dst[e] = u;
              }
            }
          }
        }
        if (valid && p.lse)
          p.lse[(size_t)h * p.total + tok] = (l > 0.f) ? (m * 0.6931471805599453f + logf(l)) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace mimo
