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
// The kernels here (warp-level mma.sync m16n8k16: bf16 in, fp32 accumulate;
// P and dS rounded to bf16 as operands):
//   bwd_preprocess_kernel  D and the sink terms, one warp per (token, head)
//   bwd_sink_kernel        dsigma_h, one CTA per head (deterministic sum)
//   bwd_dq_kernel          CTA per (128-query tile, head): loops over key tiles
//                          (double-buffered)
//   bwd_dkv_kernel<DV>     CTA per (64-key tile, KV head): loops over the
//   bwd_dkv_kernel<DK>     group's heads and query tiles (double-buffered);
//                          dV and dK in two passes (each accumulator alone
//                          fits the registers).  Used for fp32 out / dout;
//                          with bf16 ones dK and dV come from the tcgen05
//                          kernel in backward_tc_kernel.cuh.
// Tiles of 64 rows sit in shared memory with a 16-byte-chunk XOR swizzle
// (chunk ^ row % 8) so that ldmatrix reads are conflict-free.  No kernel
// here waits on another thread beyond __syncthreads.
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 7  // site numbers of the checked build

namespace mimo {

constexpr int kBwTile = 64;
constexpr int kBwQK = 192, kBwV = 128;
constexpr int kBwSmemTile192 = kBwTile * kBwQK * 2;  // 24 KB
constexpr int kBwSmemTile128 = kBwTile * kBwV * 2;   // 16 KB
constexpr int kBkThreads = 256;  // dQ and dK / dV kernels: 8 warps
constexpr int kBkStage = kBwSmemTile192 + kBwSmemTile128 + 2 * kBwTile * 4;  // Q, dO, lse, D
constexpr int kBkSmemBytes = kBwSmemTile192 + kBwSmemTile128 + 2 * kBkStage + 1024;
constexpr int kBqRows = 128;  // query rows of a dQ CTA
constexpr int kBqSmemBytes = kBqRows * (kBwQK + kBwV) * 2 + 2 * kBqRows * 4 +
                             2 * (kBwSmemTile192 + kBwSmemTile128) + 1024;

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
  int total, Hq, Hkv, G, window, num_seqs, max_seqlen;
  float scale, scale_log2, v_scale;
  int io_f32;                // out / dout are fp32
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile of `cpr` chunks per row.
__device__ __forceinline__ uint32_t bw_off(int row, int chunk, int cpr) {
  return static_cast<uint32_t>((row * cpr + (chunk ^ (row & 7))) * 16);
}

// fp32 dO rows into a swizzled bf16 tile (rows at or past `rows_valid` are
// zero); all of a thread's loads are issued before its stores.
template <int NT, int ROWS = kBwTile>
__device__ __forceinline__ void bw_load_dout_f32_tile(uint8_t* tile, const float* dout, int Hq, int h,
                                                      int row0, int rows_valid) {
  constexpr int cpr = kBwV / 8;
  constexpr int per = ROWS * cpr / NT;
  uint4 val[per];
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * NT;
    const int r = w / cpr, c = w % cpr;
    float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
    if (r < rows_valid) {
      const float4* src = reinterpret_cast<const float4*>(dout + ((size_t)(row0 + r) * Hq + h) * kBwV + c * 8);
      lo = src[0];
      hi = src[1];
    }
    val[i] = make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y),
                        pack_bf16(hi.z, hi.w));
  }
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * NT;
    *reinterpret_cast<uint4*>(tile + bw_off(w / cpr, w % cpr, cpr)) = val[i];
  }
}

// cp.async (Ampere-style asynchronous global -> shared copies); a source size
// of 0 writes zeros without reading the source.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Rows [row0, row0 + ROWS) of a [*, H, D] bf16 tensor (head `head`) into a
// swizzled tile with cp.async; rows at or past `rows_valid` are zero-filled.
template <int D, int NT, int ROWS = kBwTile>
__device__ __forceinline__ void bw_async_tile(uint8_t* tile, const __nv_bfloat16* base, int H, int head,
                                              int row0, int rows_valid) {
  constexpr int cpr = D / 8;
  constexpr int per = ROWS * cpr / NT;
  const uint32_t t = smem_u32(tile);
#pragma unroll
  for (int i = 0; i < per; ++i) {
    const int w = threadIdx.x + i * NT;
    const int r = w / cpr, c = w % cpr;
    const bool ok = r < rows_valid;
    cp_async16(t + bw_off(r, c, cpr), ok ? base + ((size_t)(row0 + r) * H + head) * D + c * 8 : base,
               ok ? 16 : 0);
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

// dQ for one 128-query tile of one head.  Eight warps of 16 query rows each
// share the key tiles, which are double-buffered with cp.async; a warp skips
// a key tile that its rows cannot see.
__global__ void __launch_bounds__(kBkThreads, 1) bwd_dq_kernel(const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t bsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsm_raw) + 1023) & ~uintptr_t(1023));
  constexpr int QR = kBqRows;
  uint8_t* sQ = sm;
  uint8_t* sdO = sQ + QR * kBwQK * 2;
  float* sL = reinterpret_cast<float*>(sdO + QR * kBwV * 2);  // lse
  float* sD = sL + QR;
  uint8_t* stages = reinterpret_cast<uint8_t*>(sD + QR);  // 2 x {K, V}
  constexpr int kStage = kBwSmemTile192 + kBwSmemTile128;

  const int h = blockIdx.y, seq = blockIdx.z;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  if (!seq_in_bounds(b0, len, p.max_seqlen, p.total)) {  // bad cu_seqlens: touch nothing
    if (threadIdx.x == 0) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int nqt = (len + QR - 1) / QR;
  if ((int)blockIdx.x >= nqt) return;
  const int qt = nqt - 1 - (int)blockIdx.x;  // the longest key loops are issued first
  const int q0 = qt * QR;
  const int g = h / p.G;
  const int qv = min(QR, len - q0);
  const int last_q = q0 + qv - 1;
  const int kt_lo = p.window > 0 ? max(0, q0 - p.window + 1) / kBwTile : 0;
  const int kt_hi = last_q / kBwTile;
  const int n_items = kt_hi - kt_lo + 1;

  auto issue = [&](int j, int st) {
    uint8_t* sK = stages + st * kStage;
    const int k0 = (kt_lo + j) * kBwTile;
    const int kv = min(kBwTile, len - k0);
    bw_async_tile<kBwQK, kBkThreads>(sK, p.k, p.Hkv, g, b0 + k0, kv);
    bw_async_tile<kBwV, kBkThreads>(sK + kBwSmemTile192, p.v, p.Hkv, g, b0 + k0, kv);
  };

  bw_async_tile<kBwQK, kBkThreads, QR>(sQ, p.q, p.Hq, h, b0 + q0, qv);
  // dO as bf16 (fp32 inputs rounded): the dP product runs in bf16
  if (p.io_f32)
    bw_load_dout_f32_tile<kBkThreads, QR>(sdO, reinterpret_cast<const float*>(p.dout), p.Hq, h, b0 + q0, qv);
  else
    bw_async_tile<kBwV, kBkThreads, QR>(sdO, reinterpret_cast<const __nv_bfloat16*>(p.dout), p.Hq, h,
                                        b0 + q0, qv);
  {
    const int r = threadIdx.x & (QR - 1);
    const float* src = (threadIdx.x < QR ? p.lse : p.D) + (size_t)h * p.total + b0 + q0;
    const bool ok = r < qv;
    cp_async4(smem_u32(sL) + threadIdx.x * 4, ok ? src + r : src, ok ? 4 : 0);
  }
  issue(0, 0);
  cp_async_commit();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = 16 * warp;  // this warp's query rows within the tile
  const int gr = lane >> 2, t4 = lane & 3;
  float dq[24][4];
#pragma unroll
  for (int n = 0; n < 24; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

  // ldmatrix lane addressing
  const int a_row = r0 + (lane & 15), a_ch = lane >> 4;                        // A: rows x 16 dims
  const int b_row = (lane & 7) + ((lane >> 4) << 3), b_ch = (lane >> 3) & 1;   // B (n-major rows)
  const int t_row = (lane & 7) + (((lane >> 3) & 1) << 3), t_ch = lane >> 4;   // B via .trans
  const uint32_t aQ = smem_u32(sQ), adO = smem_u32(sdO);
  const int qa = q0 + r0 + gr, qb = qa + 8;
  const int wq_lo = q0 + r0, wq_hi = q0 + r0 + 15;  // this warp's query positions

#pragma unroll 1
  for (int it = 0; it < n_items; ++it) {
    const int st = it & 1;
    if (it + 1 < n_items) issue(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t aK = smem_u32(stages + st * kStage), aV = aK + kBwSmemTile192;
    const int k0 = (kt_lo + it) * kBwTile;
    const bool seen = k0 <= wq_hi && wq_lo < len &&
                      (p.window == 0 || k0 + kBwTile - 1 >= wq_lo - p.window + 1);
    if (seen) {
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
        const float la = sL[r0 + gr] * 1.4426950408889634f, lb = sL[r0 + gr + 8] * 1.4426950408889634f;
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
    __syncthreads();  // stage st is free for the copies of item it + 2
  }
  cp_async_wait<0>();

  // write dq * scale for valid rows
  const int ra = r0 + gr, rb = ra + 8;
  const long long dq_rows = (long long)p.total * p.Hq;
  const bool oka = ra < qv && MIMO_ROW_OK((long long)(b0 + q0 + ra) * p.Hq + h, dq_rows);
  const bool okb = rb < qv && MIMO_ROW_OK((long long)(b0 + q0 + rb) * p.Hq + h, dq_rows);
#pragma unroll
  for (int n = 0; n < 24; ++n) {
    const int col = 8 * n + 2 * t4;
    if (oka) {
      float* dst = p.dq + ((size_t)(b0 + q0 + ra) * p.Hq + h) * kBwQK + col;
      *reinterpret_cast<float2*>(dst) = make_float2(dq[n][0] * p.scale, dq[n][1] * p.scale);
    }
    if (okb) {
      float* dst = p.dq + ((size_t)(b0 + q0 + rb) * p.Hq + h) * kBwQK + col;
      *reinterpret_cast<float2*>(dst) = make_float2(dq[n][2] * p.scale, dq[n][3] * p.scale);
    }
  }
}

// dV (kDV) or dK (!kDV) for one 64-key tile of one KV head.  Eight warps:
// warp w owns key rows 16 (w % 4) .. +15 and query half w / 4 of every query
// tile, so the two warps of a key slice split each tile's queries and add
// their partial sums once at the end.  The (head, query tile) items are
// double-buffered: the next item's Q, dO, lse and D are copied with cp.async
// while the current one is computed.
template <bool kDV>
__global__ void __launch_bounds__(kBkThreads, 1) bwd_dkv_kernel(const BackwardParams p) {
  extern __shared__ __align__(1024) uint8_t bsm_raw2[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bsm_raw2) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sm;
  uint8_t* sV = sK + kBwSmemTile192;
  uint8_t* stages = sV + kBwSmemTile128;  // 2 x {Q, dO, lse, D}

  // Key tiles in ascending order, KV heads fastest: under a causal mask the
  // longest query loops are issued first.
  const int kt = (int)blockIdx.x / p.Hkv, g = (int)blockIdx.x % p.Hkv, seq = blockIdx.y;
  const int b0 = p.cu_seqlens[seq], len = p.cu_seqlens[seq + 1] - b0;
  if (!seq_in_bounds(b0, len, p.max_seqlen, p.total)) {  // bad cu_seqlens: touch nothing
    if (threadIdx.x == 0) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int k0 = kt * kBwTile;
  if (k0 >= len) return;
  const int kv = min(kBwTile, len - k0);
  const int last_k = k0 + kv - 1;
  const int qt_lo = kt;
  const int qt_hi = p.window > 0 ? min((len - 1) / kBwTile, (last_k + p.window - 1) / kBwTile)
                                 : (len - 1) / kBwTile;
  const int nq = qt_hi - qt_lo + 1;
  const int n_items = p.G * nq;

  // item j: head g G + j / nq, query tile qt_lo + j % nq, into stage st
  auto issue = [&](int j, int st) {
    uint8_t* sQ = stages + st * kBkStage;
    const int h = g * p.G + j / nq;
    const int q0 = (qt_lo + j % nq) * kBwTile;
    const int qv = min(kBwTile, len - q0);
    bw_async_tile<kBwQK, kBkThreads>(sQ, p.q, p.Hq, h, b0 + q0, qv);
    if (p.io_f32)
      bw_load_dout_f32_tile<kBkThreads>(sQ + kBwSmemTile192, reinterpret_cast<const float*>(p.dout), p.Hq, h,
                                        b0 + q0, qv);
    else
      bw_async_tile<kBwV, kBkThreads>(sQ + kBwSmemTile192, reinterpret_cast<const __nv_bfloat16*>(p.dout),
                                      p.Hq, h, b0 + q0, qv);
    if (threadIdx.x < 2 * kBwTile) {
      const int r = threadIdx.x & (kBwTile - 1);
      const float* src = (threadIdx.x < kBwTile ? p.lse : p.D) + (size_t)h * p.total + b0 + q0;
      const bool ok = r < qv;
      cp_async4(smem_u32(sQ + kBwSmemTile192 + kBwSmemTile128) + threadIdx.x * 4, ok ? src + r : src,
                ok ? 4 : 0);
    }
  };

  bw_async_tile<kBwQK, kBkThreads>(sK, p.k, p.Hkv, g, b0 + k0, kv);
  if (!kDV) bw_async_tile<kBwV, kBkThreads>(sV, p.v, p.Hkv, g, b0 + k0, kv);
  issue(0, 0);
  cp_async_commit();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kw = 16 * (warp & 3);   // key rows of this warp
  const int qh = 32 * (warp >> 2);  // query half of this warp within each tile
  const int gr = lane >> 2, t4 = lane & 3;
  constexpr int NB = kDV ? 16 : 24;  // output n-blocks: 128 or 192 dims
  float acc[NB][4];
#pragma unroll
  for (int n = 0; n < NB; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  const int a_row = kw + (lane & 15), a_ch = lane >> 4;
  const int b_row = (lane & 7) + ((lane >> 4) << 3), b_ch = (lane >> 3) & 1;
  const int t_row = (lane & 7) + (((lane >> 3) & 1) << 3), t_ch = lane >> 4;
  const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
  const int ka = k0 + kw + gr, kb = ka + 8;  // this thread's key rows

#pragma unroll 1
  for (int it = 0; it < n_items; ++it) {
    const int st = it & 1;
    if (it + 1 < n_items) issue(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();  // this thread's copies of item `it` (and the K/V tile) have landed
    __syncthreads();     // ... and everyone's
    uint8_t* sQ = stages + st * kBkStage;
    const uint32_t aQ = smem_u32(sQ), adO = aQ + kBwSmemTile192;
    const float* sL = reinterpret_cast<const float*>(sQ + kBwSmemTile192 + kBwSmemTile128);
    const float* sD = sL + kBwTile;
    const int q0 = (qt_lo + it % nq) * kBwTile;

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
        const int qr = qh + 8 * n + 2 * t4 + (e & 1);  // query row within the tile
        const int qp = q0 + qr;
        const bool vis = qp < len && kp < len && bw_visible(qp, kp, p.window);
        const float lr = sL[qr] * 1.4426950408889634f;
        const float pr = vis ? ex2(s[n][e] * p.scale_log2 - lr) : 0.f;
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
    __syncthreads();  // stage st is free for the copies of item it + 2
  }
  cp_async_wait<0>();
  __syncthreads();

  // the second query half's partial sums, through shared memory ([warp][n e][lane])
  float* red = reinterpret_cast<float*>(stages);
  if (warp >= 4) {
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[((warp - 4) * NB * 4 + n * 4 + e) * 32 + lane] = acc[n][e];
  }
  __syncthreads();
  if (warp >= 4) return;
#pragma unroll
  for (int n = 0; n < NB; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] += red[(warp * NB * 4 + n * 4 + e) * 32 + lane];

  // write dV * v_scale or dK * scale for valid keys
  const float f = kDV ? p.v_scale : p.scale;
  constexpr int D = kDV ? kBwV : kBwQK;
  float* out = kDV ? p.dv : p.dk;
  const int ra = kw + gr, rb = ra + 8;
  const long long kv_rows = (long long)p.total * p.Hkv;
  const bool oka = ra < kv && MIMO_ROW_OK((long long)(b0 + k0 + ra) * p.Hkv + g, kv_rows);
  const bool okb = rb < kv && MIMO_ROW_OK((long long)(b0 + k0 + rb) * p.Hkv + g, kv_rows);
#pragma unroll
  for (int n = 0; n < NB; ++n) {
    const int col = 8 * n + 2 * t4;
    if (oka)
      *reinterpret_cast<float2*>(out + ((size_t)(b0 + k0 + ra) * p.Hkv + g) * D + col) =
          make_float2(acc[n][0] * f, acc[n][1] * f);
    if (okb)
      *reinterpret_cast<float2*>(out + ((size_t)(b0 + k0 + rb) * p.Hkv + g) * D + col) =
          make_float2(acc[n][2] * f, acc[n][3] * f);
  }
}

}  // namespace mimo
