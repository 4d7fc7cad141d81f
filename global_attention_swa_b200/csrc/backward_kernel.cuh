// Prefill backward: gradients of the sliding-window / global attention with a
// learnable sink (MiMo-V2-Flash model doc, "Key features": learnable
// attention-sink bias), for training.
//
// Per query head h, row i and visible key j (S = s <q, k>, lse from the
// forward, the sink included; P = exp(S - lse)):
//   D_i = <dO_i, O_i>,  dP_ij = v_scale <dO_i, v_j>,  dS_ij = P_ij (dP_ij - D_i)
//   dq_i = s sum_j dS_ij k_j;  dk_j = s sum_{h in group, i} dS_ij q_i;
//   dv_j = v_scale sum_{h in group, i} P_ij dO_i;  dsigma_h = -sum_i exp(sigma_h - lse_i) D_i
//
// Five launches, warp-level mma.sync m16n8k16 (bf16 in, fp32 accumulate; P
// and dS rounded to bf16 as operands):
//   bwd_preprocess_kernel  D and the sink terms, one warp per (token, head)
//   bwd_sink_kernel        dsigma_h, one CTA per head (deterministic sum)
//   bwd_dq_kernel          CTA per (64-query tile, head): loops over key tiles
//   bwd_dkv_kernel<DV>     CTA per (64-key tile, KV head): loops over the
//   bwd_dkv_kernel<DK>     group's heads and query tiles; dV and dK in two
//                          passes (each accumulator alone fits the registers)
// Tiles of 64 rows sit in shared memory with a 16-byte-chunk XOR swizzle
// (chunk ^ row % 8) so that ldmatrix reads are conflict-free.  No kernel
// waits on another thread beyond __syncthreads.
#pragma once

#include "common.cuh"

namespace mimo {

constexpr int kBwTile = 64;
constexpr int kBwThreads = 128;  // 4 warps x 16 rows
constexpr int kBwQK = 192, kBwV = 128;
constexpr int kBwSmemTile192 = kBwTile * kBwQK * 2;  // 24 KB
constexpr int kBwSmemTile128 = kBwTile * kBwV * 2;   // 16 KB
constexpr int kBwSmemBytes = 2 * kBwSmemTile192 + 2 * kBwSmemTile128 + 2 * kBwTile * 4 + 1024;

struct BackwardParams {
  const __nv_bfloat16* q;    // [Nt, Hq, 192]
  const __nv_bfloat16* k;    // [Nt, Hkv, 192]
  const __nv_bfloat16* v;    // [Nt, Hkv, 128]
  const void* out;           // [Nt, Hq, 128] forward output (bf16 or fp32)
  const void* dout;          // [Nt, Hq, 128] same dtype
  const float* lse;          // [Hq, Nt] natural log, sink included
  const float* sinks;        // [Hq] or null
  const int32_t* cu_seqlens;
  float* dq;                 // [Nt, Hq, 192]
  float* dk;                 // [Nt, Hkv, 192]
  float* dv;                 // [Nt, Hkv, 128]
  float* dsinks;             // [Hq] or null
  float* D;                  // [Hq, Nt] workspace
  float* psd;                // [Hq, Nt] workspace: exp(sigma - lse) * D
  int total, Hq, Hkv, G, window, num_seqs;
  float scale, scale_log2, v_scale;
  int io_f32;                // out / dout are fp32
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile of `cpr` chunks per row.
__device__ __forceinline__ uint32_t bw_off(int row, int chunk, int cpr) {
  return static_cast<uint32_t>((row * cpr + (chunk ^ (row & 7))) * 16);
}

// Load rows [row0, row0 + 64) of a [*, H, D] bf16 tensor (head `head`) into a
// swizzled tile; rows at or past `rows_valid` are zero.  All of a thread's
// loads are issued before its stores, so the tile costs one memory latency.
template <int D>
__device__ __forceinline__ void bw_load_tile(uint8_t* tile, const __nv_bfloat16* base, int H, int head,
                                             int row0, int rows_valid) {
  constexpr int cpr = D / 8;
  constexpr int per = kBwTile * cpr / kBwThreads;
  uint4 val[per];
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * kBwThreads;
    const int r = w / cpr, c = w % cpr;
    val[i] = (r < rows_valid)
                 ? *reinterpret_cast<const uint4*>(base + ((size_t)(row0 + r) * H + head) * D + c * 8)
                 : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * kBwThreads;
    *reinterpret_cast<uint4*>(tile + bw_off(w / cpr, w % cpr, cpr)) = val[i];
  }
}

// dO rows (bf16 or fp32 in memory) into a swizzled bf16 tile, loads batched as above.
__device__ __forceinline__ void bw_load_dout_tile(uint8_t* tile, const void* dout, int f32, int Hq, int h,
                                                  int row0, int rows_valid) {
  constexpr int cpr = kBwV / 8;
  constexpr int per = kBwTile * cpr / kBwThreads;  // 8
  uint4 val[per];
  if (f32) {
#pragma unroll
    for (int i = 0; i < per; ++i) {
      const int w = threadIdx.x + i * kBwThreads;
      const int r = w / cpr, c = w % cpr;
      float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
      if (r < rows_valid) {
        const float4* src = reinterpret_cast<const float4*>(
            reinterpret_cast<const float*>(dout) + ((size_t)(row0 + r) * Hq + h) * kBwV + c * 8);
        lo = src[0];
        hi = src[1];
      }
      val[i] = make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y),
                          pack_bf16(hi.z, hi.w));
    }
  } else {
#pragma unroll
    for (int i = 0; i < per; ++i) {
      const int w = threadIdx.x + i * kBwThreads;
      const int r = w / cpr, c = w % cpr;
      val[i] = (r < rows_valid)
                   ? *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(dout) +
                                                     ((size_t)(row0 + r) * Hq + h) * kBwV + c * 8)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * kBwThreads;
    *reinterpret_cast<uint4*>(tile + bw_off(w / cpr, w % cpr, cpr)) = val[i];
  }
}

__device__ __forceinline__ bool bw_visible(int qp, int kp, int window) {
  return kp <= qp && (window == 0 || qp - kp <= window - 1);
}

__device__ __forceinline__ float bw_load_io(const void* p, size_t i, int f32) {
  return f32 ? reinterpret_cast<const float*>(p)[i]
             : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

// D = <dO, O> (dO as bf16) and exp(sigma - lse) * D; one warp per (token, head), lane: 4 columns.
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BackwardParams p) {
  const long wid = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long)p.total * p.Hq) return;
  const int tok = (int)(wid / p.Hq), h = (int)(wid % p.Hq);
  const size_t base = ((size_t)tok * p.Hq + h) * kBwV + lane * 4;
  // dO rounded to bf16 as the dP products see it, so that D and dP cancel
  // exactly where they should (e.g. a row with one visible key and no sink)
  float d = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    d += bw_load_io(p.out, base + e, p.io_f32) *
         __bfloat162float(__float2bfloat16_rn(bw_load_io(p.dout, base + e, p.io_f32)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
  if (lane == 0) {
    const size_t hi = (size_t)h * p.total + tok;
    p.D[hi] = d;
    if (p.sinks) p.psd[hi] = expf(p.sinks[h] - p.lse[hi]) * d;
  }
}

// dsigma_h = -sum_i psd[h, i]: one CTA per head, fixed-order tree sum.
__global__ void __launch_bounds__(256) bwd_sink_kernel(const BackwardParams p) {
  __shared__ float part[256];
  const int h = blockIdx.x;
  float acc = 0.f;
  for (int i = threadIdx.x; i < p.total; i += blockDim.x) acc += p.psd[(size_t)h * p.total + i];
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) p.dsinks[h] = -part[0];
}

// dQ for one 64-query tile of one head.
__global__ void __launch_bounds__(kBwThreads) bwd_dq_kernel(const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t bsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm;
  uint8_t* sK = sQ + kBwSmemTile192;
  uint8_t* sdO = sK + kBwSmemTile192;
  uint8_t* sV = sdO + kBwSmemTile128;
  float* sL = reinterpret_cast<float*>(sV + kBwSmemTile128);  // lse * log2(e)
  float* sD = sL + kBwTile;

  const int qt = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  const int q0 = qt * kBwTile;
  if (q0 >= len) return;
  const int g = h / p.G;
  const int qv = min(kBwTile, len - q0);
  bw_load_tile<kBwQK>(sQ, p.q, p.Hq, h, b0 + q0, qv);
  // dO as bf16 (fp32 inputs rounded): the dP product runs in bf16
  bw_load_dout_tile(sdO, p.dout, p.io_f32, p.Hq, h, b0 + q0, qv);
  for (int r = threadIdx.x; r < kBwTile; r += blockDim.x) {
    const bool ok = r < qv;
    sL[r] = ok ? p.lse[(size_t)h * p.total + b0 + q0 + r] * 1.4426950408889634f : 0.f;
    sD[r] = ok ? p.D[(size_t)h * p.total + b0 + q0 + r] : 0.f;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = warp * 16;                // this warp's query rows within the tile
  const int gr = lane >> 2, t4 = lane & 3;
  float dq[24][4];
#pragma unroll
  for (int n = 0; n < 24; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

  const int last_q = q0 + qv - 1;
  const int kt_lo = p.window > 0 ? max(0, q0 - p.window + 1) / kBwTile : 0;
  const int kt_hi = last_q / kBwTile;
  // ldmatrix lane addressing
  const int a_row = r0 + (lane & 15), a_ch = lane >> 4;                        // A: rows x 16 dims
  const int b_row = (lane & 7) + ((lane >> 4) << 3), b_ch = (lane >> 3) & 1;   // B (n-major rows)
  const int t_row = (lane & 7) + (((lane >> 3) & 1) << 3), t_ch = lane >> 4;   // B via .trans
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), adO = smem_u32(sdO), aV = smem_u32(sV);
  for (int kt = kt_lo; kt <= kt_hi; ++kt) {
    const int k0 = kt * kBwTile;
    __syncthreads();  // previous tile's readers are done (and the row data above is visible)
    bw_load_tile<kBwQK>(sK, p.k, p.Hkv, g, b0 + k0, min(kBwTile, len - k0));
    bw_load_tile<kBwV>(sV, p.v, p.Hkv, g, b0 + k0, min(kBwTile, len - k0));
    __syncthreads();
    // S = Q K^T (16 rows x 64 keys)
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
      uint32_t a[4];
      ldsm_x4(aQ + bw_off(a_row, 2 * kk + a_ch, 24), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        uint32_t b[4];
        ldsm_x4(aK + bw_off(16 * nb + b_row, 2 * kk + b_ch, 24), b[0], b[1], b[2], b[3]);
        mma_bf16_16816(s[2 * nb], a, b[0], b[1]);
        mma_bf16_16816(s[2 * nb + 1], a, b[2], b[3]);
      }
    }
    // dP = dO V^T (16 x 64)
    float dp[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldsm_x4(adO + bw_off(a_row, 2 * kk + a_ch, 16), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        uint32_t b[4];
        ldsm_x4(aV + bw_off(16 * nb + b_row, 2 * kk + b_ch, 16), b[0], b[1], b[2], b[3]);
        mma_bf16_16816(dp[2 * nb], a, b[0], b[1]);
        mma_bf16_16816(dp[2 * nb + 1], a, b[2], b[3]);
      }
    }
    // P and dS = P (v_scale dP - D), as bf16 A fragments for dS K
    uint32_t ds[4][4];  // [k-step of 16 keys][A register]
    {
      const int qa = q0 + r0 + gr, qb = qa + 8;
      const float la = sL[r0 + gr], lb = sL[r0 + gr + 8];
      const float Da = sD[r0 + gr], Db = sD[r0 + gr + 8];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        float d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qp = (e < 2) ? qa : qb;
          const int kp = k0 + 8 * n + 2 * t4 + (e & 1);
          const bool vis = qp < len && kp < len && bw_visible(qp, kp, p.window);
          const float pr = vis ? ex2(s[n][e] * p.scale_log2 - ((e < 2) ? la : lb)) : 0.f;
          d[e] = pr * (p.v_scale * dp[n][e] - ((e < 2) ? Da : Db));
        }
        // n-block n covers keys 8n..8n+7: A registers {0,1} of k-step n/2 (n even) or {2,3} (odd)
        ds[n >> 1][(n & 1) * 2 + 0] = pack_bf16(d[0], d[1]);
        ds[n >> 1][(n & 1) * 2 + 1] = pack_bf16(d[2], d[3]);
      }
    }
    // dQ += dS K (16 x 192): k = keys, B from K rows via ldmatrix.trans
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int np = 0; np < 12; ++np) {
        uint32_t b[4];
        ldsm_x4_t(aK + bw_off(16 * ks + t_row, 2 * np + t_ch, 24), b[0], b[1], b[2], b[3]);
        mma_bf16_16816(dq[2 * np], ds[ks], b[0], b[1]);
        mma_bf16_16816(dq[2 * np + 1], ds[ks], b[2], b[3]);
      }
    }
  }
  // write dq * scale for valid rows
  const int ra = r0 + gr, rb = ra + 8;
#pragma unroll
  for (int n = 0; n < 24; ++n) {
    const int col = 8 * n + 2 * t4;
    if (ra < qv) {
      float* dst = p.dq + ((size_t)(b0 + q0 + ra) * p.Hq + h) * kBwQK + col;
      *reinterpret_cast<float2*>(dst) = make_float2(dq[n][0] * p.scale, dq[n][1] * p.scale);
    }
    if (rb < qv) {
      float* dst = p.dq + ((size_t)(b0 + q0 + rb) * p.Hq + h) * kBwQK + col;
      *reinterpret_cast<float2*>(dst) = make_float2(dq[n][2] * p.scale, dq[n][3] * p.scale);
    }
  }
}

// dV (kDV) or dK (!kDV) for one 64-key tile of one KV head.
template <bool kDV>
__global__ void __launch_bounds__(kBwThreads) bwd_dkv_kernel(const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t bsm_raw2[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsm_raw2) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sm;
  uint8_t* sQ = sK + kBwSmemTile192;
  uint8_t* sV = sQ + kBwSmemTile192;
  uint8_t* sdO = sV + kBwSmemTile128;
  float* sL = reinterpret_cast<float*>(sdO + kBwSmemTile128);
  float* sD = sL + kBwTile;

  const int kt = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  const int k0 = kt * kBwTile;
  if (k0 >= len) return;
  const int kv = min(kBwTile, len - k0);
  bw_load_tile<kBwQK>(sK, p.k, p.Hkv, g, b0 + k0, kv);
  if (!kDV) bw_load_tile<kBwV>(sV, p.v, p.Hkv, g, b0 + k0, kv);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kw = warp * 16;
  const int gr = lane >> 2, t4 = lane & 3;
  constexpr int NB = kDV ? 16 : 24;  // output n-blocks: 128 or 192 dims
  float acc[NB][4];
#pragma unroll
  for (int n = 0; n < NB; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  const int last_k = k0 + kv - 1;
  const int qt_lo = k0 / kBwTile;
  const int qt_hi = p.window > 0 ? min((len - 1) / kBwTile, (last_k + p.window - 1) / kBwTile)
                                 : (len - 1) / kBwTile;
  const int a_row = kw + (lane & 15), a_ch = lane >> 4;
  const int b_row = (lane & 7) + ((lane >> 4) << 3), b_ch = (lane >> 3) & 1;
  const int t_row = (lane & 7) + (((lane >> 3) & 1) << 3), t_ch = lane >> 4;
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), adO = smem_u32(sdO), aV = smem_u32(sV);
  const int ka = k0 + kw + gr, kb = ka + 8;  // this thread's key rows

  for (int hh = 0; hh < p.G; ++hh) {
    const int h = g * p.G + hh;
    for (int qt = qt_lo; qt <= qt_hi; ++qt) {
      const int q0 = qt * kBwTile;
      const int qv = min(kBwTile, len - q0);
      __syncthreads();
      bw_load_tile<kBwQK>(sQ, p.q, p.Hq, h, b0 + q0, qv);
      bw_load_dout_tile(sdO, p.dout, p.io_f32, p.Hq, h, b0 + q0, qv);
      for (int r = threadIdx.x; r < kBwTile; r += blockDim.x) {
        const bool ok = r < qv;
        sL[r] = ok ? p.lse[(size_t)h * p.total + b0 + q0 + r] * 1.4426950408889634f : 0.f;
        sD[r] = ok ? p.D[(size_t)h * p.total + b0 + q0 + r] : 0.f;
      }
      __syncthreads();
      // The 64 queries in two halves of 32 (keeps the temporaries small next to
      // the 16 x 192 dK accumulator).
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        const int qh = 32 * hf;  // first query row of this half within the tile
        // S^T = K Q^T (16 keys x 32 queries)
        float s[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          uint32_t a[4];
          ldsm_x4(aK + bw_off(a_row, 2 * kk + a_ch, 24), a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            uint32_t b[4];
            ldsm_x4(aQ + bw_off(qh + 16 * nb + b_row, 2 * kk + b_ch, 24), b[0], b[1], b[2], b[3]);
            mma_bf16_16816(s[2 * nb], a, b[0], b[1]);
            mma_bf16_16816(s[2 * nb + 1], a, b[2], b[3]);
          }
        }
        float dp[4][4];
        if (!kDV) {
          // dP^T = V dO^T (16 keys x 32 queries)
#pragma unroll
          for (int n = 0; n < 4; ++n) dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t a[4];
            ldsm_x4(aV + bw_off(a_row, 2 * kk + a_ch, 16), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              uint32_t b[4];
              ldsm_x4(adO + bw_off(qh + 16 * nb + b_row, 2 * kk + b_ch, 16), b[0], b[1], b[2], b[3]);
              mma_bf16_16816(dp[2 * nb], a, b[0], b[1]);
              mma_bf16_16816(dp[2 * nb + 1], a, b[2], b[3]);
            }
          }
        }
        // P^T (kDV) or dS^T (!kDV) as bf16 A fragments: k = queries
        uint32_t af[2][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          float d[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kp = (e < 2) ? ka : kb;
            const int qr = qh + 8 * n + 2 * t4 + (e & 1);   // query row within the tile
            const int qp = q0 + qr;
            const bool vis = qp < len && kp < len && bw_visible(qp, kp, p.window);
            const float pr = vis ? ex2(s[n][e] * p.scale_log2 - sL[qr]) : 0.f;
            d[e] = kDV ? pr : pr * (p.v_scale * dp[n][e] - sD[qr]);
          }
          af[n >> 1][(n & 1) * 2 + 0] = pack_bf16(d[0], d[1]);
          af[n >> 1][(n & 1) * 2 + 1] = pack_bf16(d[2], d[3]);
        }
        // acc += af (16 keys x 32 queries) x [dO | Q] (32 queries x 128 | 192 dims)
        const uint32_t aB = kDV ? adO : aQ;
        constexpr int cpr = kDV ? 16 : 24;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
          for (int np = 0; np < NB / 2; ++np) {
            uint32_t b[4];
            ldsm_x4_t(aB + bw_off(qh + 16 * ks + t_row, 2 * np + t_ch, cpr), b[0], b[1], b[2], b[3]);
            mma_bf16_16816(acc[2 * np], af[ks], b[0], b[1]);
            mma_bf16_16816(acc[2 * np + 1], af[ks], b[2], b[3]);
          }
        }
      }
    }
  }
  // write dV * v_scale or dK * scale for valid keys
  const float f = kDV ? p.v_scale : p.scale;
  constexpr int D = kDV ? kBwV : kBwQK;
  float* out = kDV ? p.dv : p.dk;
  const int ra = kw + gr, rb = ra + 8;
#pragma unroll
  for (int n = 0; n < NB; ++n) {
    const int col = 8 * n + 2 * t4;
    if (ra < kv)
      *reinterpret_cast<float2*>(out + ((size_t)(b0 + k0 + ra) * p.Hkv + g) * D + col) =
          make_float2(acc[n][0] * f, acc[n][1] * f);
    if (rb < kv)
      *reinterpret_cast<float2*>(out + ((size_t)(b0 + k0 + rb) * p.Hkv + g) * D + col) =
          make_float2(acc[n][2] * f, acc[n][3] * f);
  }
}

}  // namespace mimo
