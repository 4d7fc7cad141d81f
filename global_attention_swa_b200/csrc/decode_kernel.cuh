// Decode: one query token per sequence against a KV cache (global linear
// cache or sliding-window ring), split over the key axis.
//
// MiMo-V2-Flash model doc: MiMoV2FlashModel.forward, `past_key_values` (only
// the new token is fed after the first call) and the "Key features" hybrid
// attention bullet (SWA layers keep only the window; the learnable sink).
//
// Work unit = (sequence b, key/value head g, split c).  The G <= 16 query heads
// that share head g are packed as the M = 16 rows of a warp-level
// mma.sync.m16n8k16 (bf16 in, fp32 accumulate): the 16 heads read every K/V
// byte once, which is what makes this step HBM-bound rather than bound by
// scalar FMA throughput (16 flop per cache byte).
//
// Pipeline per CTA: warp 4 streams 64-key K/V tiles (K: 3 boxes of 64 dims,
// V: 2 boxes, 128-byte swizzle) into a ring of kStages shared-memory stages
// with TMA; warps 0-3 each take 16 keys of every tile, compute scores,
// update an online softmax in base 2 and accumulate P.V in registers.  The
// four warps merge at the end.  With one split the sink is folded in and the
// result written out; otherwise (o, m, l) partials go to the workspace and
// decode_combine_kernel merges them with the sink.
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 3  // site numbers of the checked build

namespace mimo {

constexpr int kDecTileKeys = 64;
constexpr int kDecStages = 4;                        // long caches: one CTA per SM
constexpr int kDecShortStages = 2;                   // short caches (rings): two CTAs per SM
constexpr int kDecShortKeys = 256;                   // "short": at most this many visible slots
constexpr int kDecKBytes = kDecTileKeys * 192 * 2;   // 24576
constexpr int kDecVBytes = kDecTileKeys * 128 * 2;   // 16384
constexpr int kDecStageBytes = kDecKBytes + kDecVBytes;
constexpr int kDecThreads = 160;                     // 4 consumer warps + 1 producer warp
constexpr int kDecQRow = 400;                        // Q tile row stride (384 B + 16: ldmatrix rows on distinct banks)
constexpr int kDecQBytes = 16 * kDecQRow;
constexpr int dec_smem_bytes(int stages, int tile_rows = kDecTileKeys) {
  return stages * 5 * tile_rows * 128 + 128 /*barriers*/ + kDecQBytes + 1024 /*align*/;
}
// The end-of-split merge reuses the stage ring: [4 warps][16 rows][kDecORow]
// partial O (rows padded so that neither the fragment writes nor the row
// reads pile onto a few banks), then 3 x [4][16] floats (max, sum, rounded sum).
constexpr int kDecORow = 136;
constexpr int kDecMergeBytes = 4 * 16 * kDecORow * 4 + 3 * 4 * 16 * 4;
constexpr int kDecRingStages = 3;                    // small rings: the whole ring in flight
constexpr int kDecRingRows = 48;                     // rows of a ring tile (3 x 48 >= 129 slots)
static_assert(kDecMergeBytes <= kDecRingStages * 5 * kDecRingRows * 128, "merge buffer fits");
constexpr int kDecSmemBytes = dec_smem_bytes(kDecStages);
static_assert(kDecMergeBytes <= kDecShortStages * kDecStageBytes, "merge buffer fits");

struct DecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, 192]
  const int32_t* seqlens;  // [B]
  const float* sinks;      // [Hq] or null
  void* out;               // [B, Hq, 128]
  float* lse;              // [B, Hq] or null
  float* ws_o;             // [B*Hkv*nsplit, 16, 128]
  float* ws_ml;            // [B*Hkv*nsplit, 16, 4]: max, sum, sum of the rounded P, unused
  int B, C, Hq, Hkv, G;
  int window;
  int ring;     // 1: ring cache (C == window)
  int chunk;    // keys per split, multiple of 64
  int nsplit;   // splits per (b, g)
  int tile;     // keys per tile (rows of the K / V TMA boxes): 64, or at most 48 for a small ring
  int spec_tiles;  // > 0: stream this many tiles from slot 0 without waiting for the length (small rings)
  float scale_log2;  // softmax_scale * log2(e)
  float v_scale;
  int out_f32;
  const float* k_scale;     // [Hkv] FP8 caches only: K value = code * k_scale[g]
  const float* kv_v_scale;  // [Hkv] FP8 caches only: V value = code * kv_v_scale[g]; null = 1
};

// Visible slot range [lo, hi) of sequence b (see mimo_attn.h).
__device__ __forceinline__ void decode_range(const DecodeParams& p, int L, int& lo, int& hi) {
  if (L < 0) {
    record_status(1 /* MIMO_ERR_INVALID_ARG */);
    L = 0;
  }
  if (p.ring) {
    lo = 0;
    hi = min(L, p.C);
  } else {
    if (L > p.C) {
      record_status(1 /* MIMO_ERR_INVALID_ARG */);
      L = p.C;
    }
    hi = L;
    lo = p.window > 0 ? max(0, L - p.window) : 0;
  }
}

// kStages shared-memory stages of one K/V tile of at most kTileRows keys each
// (p.tile keys, the rows of the TMA boxes); kCtasPerSm CTAs resident per SM.
// Long caches stream 64-key tiles through 4 stages at one CTA per SM.  Short
// caches have little to pipeline: two CTAs per SM let all of a batch's units
// run in one wave, and a small ring (at most 3 x 48 slots, e.g. 129) is
// loaded whole, in three tiles issued at once without waiting for the
// sequence length (a ring's visible slots always start at slot 0; the length
// only masks keys).
template <int kStages, int kCtasPerSm, int kTileRows>
__global__ void __launch_bounds__(kDecThreads, kCtasPerSm)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t dsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr int kBox = kTileRows * 128;          // one [rows][64 dims] swizzled box
  constexpr int kStageBytes = 5 * kBox;          // K: 3 boxes, V: 2 boxes
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* q_full = empty + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(q_full + 1);
  volatile int* never_flag = abort_flag + 1;  // never raised: bounds the drains by time alone
  uint8_t* sq = smem + kStages * kStageBytes + 128;  // [16 rows][kDecQRow] Q tile

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int lo, hi;
  decode_range(p, p.seqlens[b], lo, hi);
  const int s0 = lo + split * p.chunk;
  const int s1 = min(hi, s0 + p.chunk);
  if (p.nsplit > 1 && s0 >= s1) return;  // empty split: the combine skips it
  const int nkeys = max(0, s1 - s0);

  if (threadIdx.x == 128) {  // the producer lane
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(q_full, 1);
    *never_flag = 0;
    fence_mbar_init();
    // The G query rows of this KV head: one bulk copy per 384-byte row, into
    // rows kDecQRow apart (rows >= G are never read into a fragment).
    const bool q_ok = MIMO_ROW_OK((long long)b * p.Hq + (long long)(g + 1) * p.G - 1, (long long)p.B * p.Hq);
    mbar_arrive_expect_tx(q_full, q_ok ? p.G * 384 : 0);
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + (size_t)g * p.G) * 192;
    if (q_ok)
      for (int r = 0; r < p.G; ++r) bulk_load(sq + r * kDecQRow, qg + r * 192, 384, q_full);
  }
  if (threadIdx.x == 0) {
    // sampled once, so every thread of the CTA sees the same decision
    *abort_flag = timed_out_before() ? 1 : 0;
  }
  __syncthreads();
  // after a recorded timeout elsewhere, return at entry: nothing is written
  // (the Q rows requested above land before the CTA leaves)
  if (*abort_flag) {
    if (threadIdx.x == 128) {
      drain_armed(q_full, 1, never_flag);
    }
    return;
  }
  const int tile = p.tile;
  // tiles streamed: those holding the unit's keys, or every tile of a small ring
  const int ntiles = p.spec_tiles > 0 ? p.spec_tiles : (nkeys + tile - 1) / tile;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int row0 = b * p.C + s0;
      int armed = 0;  // tiles whose loads were issued (stage t % kStages)
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % kStages;
        if (t >= kStages) {
          if (!wait_bounded(&empty[st], ((t / kStages) - 1) & 1, abort_flag)) break;
        }
        uint8_t* kb = smem + st * kStageBytes;
        uint8_t* vb = kb + 3 * kBox;
        mbar_arrive_expect_tx(&full[st], 5 * tile * 128);
        ++armed;
        const int y = row0 + t * tile;
#pragma unroll
        for (int c = 0; c < 3; ++c) tma_load_2d(kb + c * kBox, &tm_k, &full[st], g * 192 + c * 64, y);
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_2d(vb + c * kBox, &tm_v, &full[st], g * 128 + c * 64, y);
      }
      // the CTA never exits with these copies in flight (after a timed-out
      // wait the consumers may have stopped waiting for them)
      for (int s = 0; s < kStages; ++s)
        drain_armed(&full[s], armed > s ? (armed - 1 - s) / kStages + 1 : 0, never_flag);
      drain_armed(q_full, 1, never_flag);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int r0 = lane >> 2;        // rows (heads) r0 and r0 + 8
    const int cq = (lane & 3) * 2;   // column pair within an 8-wide block
    // Q fragments for all 12 k-steps of 16 dims (ldmatrix.x4: lanes 0-15 give
    // rows 0-15 at dims +0, lanes 16-31 the same rows at dims +8); rows >= G are zero.
    uint32_t qa[12][4];
    {
      const bool v0 = r0 < p.G, v1 = r0 + 8 < p.G;
      if (!wait_bounded(q_full, 0, abort_flag)) return;
      const uint32_t qrow = smem_u32(sq) + (lane & 15) * kDecQRow + (lane >> 4) * 16;
#pragma unroll
      for (int kk = 0; kk < 12; ++kk) {
        ldsm_x4(qrow + kk * 32, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        if (!v0) qa[kk][0] = qa[kk][2] = 0u;
        if (!v1) qa[kk][1] = qa[kk][3] = 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;  // running max (base 2) for rows r0, r0+8
    float l0 = 0.f, l1 = 0.f;              // per-thread partial sums (lse)
    float lr0 = 0.f, lr1 = 0.f;            // the same over the rounded P (output normaliser)

    const int kw = warp * 16;  // this warp's 16 keys within each tile
    const uint32_t sbase = smem_u32(smem);
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % kStages;
      if (!wait_bounded(&full[st], (t / kStages) & 1, abort_flag)) break;
      const int valid = min(tile, nkeys - t * tile);  // may be <= 0 for a ring's spare tile
      if (kw < valid) {
        const uint32_t kb = sbase + st * kStageBytes;
        const uint32_t vb = kb + 3 * kBox;
        // ---- S = Q K^T for keys kw .. kw+15 (two n-blocks of 8)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          // ldmatrix.x4 rows: lanes 0-7 keys kw+0..7 dims +0; 8-15 keys kw+0..7 dims +8;
          // 16-23 keys kw+8..15 dims +0; 24-31 keys kw+8..15 dims +8.
          const int krow = kw + (lane & 7) + ((lane >> 4) << 3);
          const int kcol = ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int kk = 0; kk < 12; ++kk) {
            const int c = kk >> 2;                       // 64-dim box
            const int col = (kk & 3) * 16 + kcol;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + c * kBox + sw128_offset(krow, col), b0, b1, b2, b3);
            mma_bf16_16816(s[0], qa[kk], b0, b1);
            mma_bf16_16816(s[1], qa[kk], b2, b3);
          }
        }
        // ---- scale to base 2 and mask keys past the split's end
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = kw + n * 8 + cq + e;
            const bool ok = key < valid;
            s[n][e] = ok ? s[n][e] * p.scale_log2 : -INFINITY;
            s[n][2 + e] = ok ? s[n][2 + e] * p.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, s[n][e]);
            mx1 = fmaxf(mx1, s[n][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        // mn is finite: this warp has at least one valid key in the tile
        const float a0 = ex2(m0 - mn0), a1 = ex2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        uint32_t pa[4];
        {
          float p00 = ex2(s[0][0] - mn0), p01 = ex2(s[0][1] - mn0);
          float p02 = ex2(s[0][2] - mn1), p03 = ex2(s[0][3] - mn1);
          float p10 = ex2(s[1][0] - mn0), p11 = ex2(s[1][1] - mn0);
          float p12 = ex2(s[1][2] - mn1), p13 = ex2(s[1][3] - mn1);
          pa[0] = pack_bf16(p00, p01);
          pa[1] = pack_bf16(p02, p03);
          pa[2] = pack_bf16(p10, p11);
          pa[3] = pack_bf16(p12, p13);
          l0 = l0 * a0 + ((p00 + p01) + (p10 + p11));
          l1 = l1 * a1 + ((p02 + p03) + (p12 + p13));
          lr0 = lr0 * a0 + ((bf16_lo(pa[0]) + bf16_hi(pa[0])) + (bf16_lo(pa[2]) + bf16_hi(pa[2])));
          lr1 = lr1 * a1 + ((bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3])));
        }
        // rescale O only when some row's running max moved (2^0 is exactly 1)
        if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            o[n][0] *= a0;
            o[n][1] *= a0;
            o[n][2] *= a1;
            o[n][3] *= a1;
          }
        }
        // ---- O += P V.  ldmatrix.trans rows: lanes 0-7 keys kw+0..7, 8-15 keys kw+8..15
        // (dims +0), 16-23 keys kw+0..7, 24-31 keys kw+8..15 (dims +8).
        const int vrow = kw + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int vcol = (lane >> 4) * 8;
        const bool partial = (kw + 16 > valid);
        // keys held by this thread in the V fragments: kw+cq+{0,1} (b0) and kw+8+cq+{0,1} (b1)
        const uint32_t mk0 = (kw + cq < valid ? 0x0000FFFFu : 0u) | (kw + cq + 1 < valid ? 0xFFFF0000u : 0u);
        const uint32_t mk1 = (kw + 8 + cq < valid ? 0x0000FFFFu : 0u) | (kw + 9 + cq < valid ? 0xFFFF0000u : 0u);
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          const int c = n2 >> 2;  // 64-dim box
          const int col = (n2 & 3) * 16 + vcol;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + c * kBox + sw128_offset(vrow, col), b0, b1, b2, b3);
          if (partial) {  // invalid slots may hold anything: zero them
            b0 &= mk0; b1 &= mk1; b2 &= mk0; b3 &= mk1;
          }
          mma_bf16_16816(o[2 * n2], pa, b0, b1);
          mma_bf16_16816(o[2 * n2 + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // ---- reduce l over the quad; merge the 4 warps through shared memory
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    lr0 += __shfl_xor_sync(0xffffffffu, lr0, 1);
    lr0 += __shfl_xor_sync(0xffffffffu, lr0, 2);
    lr1 += __shfl_xor_sync(0xffffffffu, lr1, 1);
    lr1 += __shfl_xor_sync(0xffffffffu, lr1, 2);
    asm volatile("bar.sync 1, 128;" ::: "memory");  // all consumers done with the stages
    float* so = reinterpret_cast<float*>(smem);      // [4 warps][16 rows][kDecORow]
    float* sm = so + 4 * 16 * kDecORow;              // [4][16] max
    float* sl = sm + 4 * 16;                         // [4][16] sum
    float* slr = sl + 4 * 16;                        // [4][16] sum of the rounded P
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = n * 8 + cq;
      *reinterpret_cast<float2*>(so + (warp * 16 + r0) * kDecORow + col) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(so + (warp * 16 + r0 + 8) * kDecORow + col) = make_float2(o[n][2], o[n][3]);
    }
    if ((lane & 3) == 0) {
      sm[warp * 16 + r0] = m0;
      sm[warp * 16 + r0 + 8] = m1;
      sl[warp * 16 + r0] = l0;
      sl[warp * 16 + r0 + 8] = l1;
      slr[warp * 16 + r0] = lr0;
      slr[warp * 16 + r0 + 8] = lr1;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // 128 threads: thread -> (row = tid / 8; columns 4 (tid & 7) + 32 j, j = 0..3,
    // so that the 8 threads of a row read 128 contiguous bytes per access)
    const int tid = threadIdx.x;
    const int row = tid >> 3;
    const int cb = (tid & 7) * 4;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w * 16 + row]);
    float wgt[4];
    float Ls = 0.f, Lrs = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      wgt[w] = (M == -INFINITY) ? 0.f : ex2(sm[w * 16 + row] - M);
      Ls += wgt[w] * sl[w * 16 + row];
      Lrs += wgt[w] * slr[w * 16 + row];
    }
    float4 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(so + (w * 16 + row) * kDecORow + cb + 32 * j);
        a.x += wgt[w] * v.x;
        a.y += wgt[w] * v.y;
        a.z += wgt[w] * v.z;
        a.w += wgt[w] * v.w;
      }
      acc[j] = a;
    }
    if (row < p.G &&
        (p.nsplit == 1 ? MIMO_ROW_OK((long long)b * p.Hq + g * p.G + row, (long long)p.B * p.Hq)
                       : MIMO_ROW_OK(((long long)b * p.Hkv + g) * p.nsplit + split, (long long)p.B * p.Hkv * p.nsplit))) {
      const int h = g * p.G + row;
      if (p.nsplit == 1) {
        // fold the sink: it joins the normaliser only
        const float sg = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
        const float Mf = fmaxf(M, sg);
        float scl = 0.f, Lf = 0.f, Lrf = 0.f;
        if (Mf != -INFINITY) {
          scl = (M == -INFINITY) ? 0.f : ex2(M - Mf);
          const float ps = (sg == -INFINITY) ? 0.f : ex2(sg - Mf);
          Lf = Ls * scl + ps;
          Lrf = Lrs * scl + ps;
        }
        const float f = (Lrf > 0.f) ? p.v_scale * scl / Lrf : 0.f;
        const size_t ob = ((size_t)b * p.Hq + h) * 128 + cb;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (p.out_f32) {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + ob + 32 * j) =
                make_float4(acc[j].x * f, acc[j].y * f, acc[j].z * f, acc[j].w * f);
          } else {
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob + 32 * j) =
                make_uint2(pack_bf16(acc[j].x * f, acc[j].y * f), pack_bf16(acc[j].z * f, acc[j].w * f));
          }
        }
        if (p.lse && (tid & 7) == 0)
          p.lse[(size_t)b * p.Hq + h] = (Lf > 0.f) ? (Mf * 0.6931471805599453f + logf(Lf)) : -INFINITY;
      } else {
        const size_t unit = ((size_t)b * p.Hkv + g) * p.nsplit + split;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float4*>(p.ws_o + (unit * 16 + row) * 128 + cb + 32 * j) = acc[j];
        if ((tid & 7) == 0) {
          p.ws_ml[(unit * 16 + row) * 4 + 0] = M;
          p.ws_ml[(unit * 16 + row) * 4 + 1] = Ls;
          p.ws_ml[(unit * 16 + row) * 4 + 2] = Lrs;
        }
      }
    }
  }
}

// Merge the split partials of every (b, query head) and fold the sink:
//   M = max(sigma, max_c m_c),  Z = 2^(sigma-M) + sum_c 2^(m_c-M) l_c,
//   out = v_scale * sum_c 2^(m_c-M) o_c / Z~,   lse = ln Z + M ln 2
// where Z~ is Z over the splits' sums of the rounded P (the values their P.V used)
// (times the V scale of the KV head for FP8 caches, whose partials are in code units).
// One warp per (b, h); lane handles 4 of the 128 value columns.
__global__ void __launch_bounds__(256)
    decode_combine_kernel(const DecodeParams p) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= p.B * p.Hq || timed_out_before()) return;  // after a recorded timeout: write nothing
  const int b = wid / p.Hq, h = wid % p.Hq;
  const int g = h / p.G, row = h % p.G;
  int lo, hi;
  decode_range(p, p.seqlens[b], lo, hi);
  int nused = min(p.nsplit, max(0, (hi - lo + p.chunk - 1) / p.chunk));
  const size_t unit0 = ((size_t)b * p.Hkv + g) * p.nsplit;
  if (nused > 0 && !MIMO_ROW_OK(unit0 + nused - 1, (long long)p.B * p.Hkv * p.nsplit)) nused = 0;
  if (!MIMO_ROW_OK((long long)b * p.Hq + h, (long long)p.B * p.Hq)) return;
  const float sg = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
  float M = sg;
  for (int c = 0; c < nused; ++c) M = fmaxf(M, p.ws_ml[((unit0 + c) * 16 + row) * 4]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Z = 0.f, Zr = 0.f;
  if (M != -INFINITY) {
    Z = (sg == -INFINITY) ? 0.f : ex2(sg - M);
    Zr = Z;
    for (int c = 0; c < nused; ++c) {
      const float4 ml = *reinterpret_cast<const float4*>(p.ws_ml + ((unit0 + c) * 16 + row) * 4);
      const float mc = ml.x;
      const float w = (mc == -INFINITY) ? 0.f : ex2(mc - M);
      Z += w * ml.y;
      Zr += w * ml.z;
      const float4 oc = reinterpret_cast<const float4*>(p.ws_o + ((unit0 + c) * 16 + row) * 128)[lane];
      acc.x += w * oc.x;
      acc.y += w * oc.y;
      acc.z += w * oc.z;
      acc.w += w * oc.w;
    }
  }
  const float vs = p.kv_v_scale ? p.kv_v_scale[g] : 1.f;
  const float f = (Zr > 0.f) ? p.v_scale * vs / Zr : 0.f;
  const size_t ob = ((size_t)b * p.Hq + h) * 128 + lane * 4;
  if (p.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + ob) =
        make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
  } else {
    uint2 u;
    u.x = pack_bf16(acc.x * f, acc.y * f);
    u.y = pack_bf16(acc.z * f, acc.w * f);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob) = u;
  }
  if (p.lse && lane == 0)
    p.lse[(size_t)b * p.Hq + h] = (Z > 0.f) ? (M * 0.6931471805599453f + logf(Z)) : -INFINITY;
}

}  // namespace mimo
