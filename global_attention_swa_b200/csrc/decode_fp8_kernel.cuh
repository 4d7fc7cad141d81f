// Decode against an FP8 (e4m3) KV cache with one scale per key/value head.
//
// MiMo-V2-Flash model doc: MiMoV2FlashModel.forward (`past_key_values`) and
// "Key features" (hybrid attention with a learnable sink; FP8 mixed
// precision).  A cache element's value is code * scale[g]: e4m3 is the OCP
// 8-bit float with 4 exponent bits (bias 7), 3 mantissa bits, no infinities
// and NaN = S.1111.111, so K and V move half the bytes of a bf16 cache.
//
// Same work split and pipeline as decode_split_kernel: unit = (sequence b,
// KV head g, split c); warp 4 streams 64-key tiles into a ring of stages with
// TMA (K: 3 boxes of 64 bytes, V: 2 boxes, 64-byte swizzle); warps 0-3 take
// 16 keys each with mma.sync.m16n8k16 in f16 (e4m3 -> f16 is exact; the
// query is rounded to f16 once, P to f16 per tile), fp32 accumulate.
//
// Fragment order.  ldmatrix on byte data hands each thread 4 consecutive
// bytes of a 16-byte row: dims 4t..4t+3 of one key (t = lane % 4).  The MMA
// reads them as k = {2t, 2t+1} (low pair) and {2t+8, 2t+9} (high pair), so
// the query fragment is loaded with the same map (k = 2t+e <-> dim 4t+e,
// k = 2t+8+e <-> dim 4t+2+e); a dot product does not depend on the order.
// For P.V, ldmatrix.trans hands a thread bytes (key 2t', dims 2c, 2c+1) and
// (key 2t'+1, same dims); one byte permute yields the f16 pairs of dim 2c and
// of dim 2c+1, so one MMA covers the even dims of a 16-dim block and a second
// the odd dims, and each thread ends with 4 consecutive output dims.
#pragma once

#include "decode_kernel.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 4  // site numbers of the checked build

namespace mimo {

constexpr int kD8TileKeys = 64;
constexpr int kD8Stages = 4;
constexpr int kD8CtasPerSm = 2;                // two CTAs (8 consumer warps) per SM hide the
                                               // per-tile latency a 20 KB tile no longer covers
constexpr int kD8KBytes = kD8TileKeys * 192;   // 12288: 3 boxes of [64 keys][64 B]
constexpr int kD8VBytes = kD8TileKeys * 128;   // 8192: 2 boxes
constexpr int kD8StageBytes = kD8KBytes + kD8VBytes;
constexpr int kD8BoxBytes = kD8TileKeys * 64;  // 4096
constexpr int kD8Threads = 160;                // 4 consumer warps + 1 producer warp
constexpr int kD8SmemBytes = kD8Stages * kD8StageBytes + 1024 /*align*/ + 256 /*barriers*/;
static_assert(4 * 16 * 128 * 4 + 3 * 4 * 16 * 4 <= kD8Stages * kD8StageBytes, "merge buffer fits");

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
  return pack_f16(bf16_lo(u), bf16_hi(u));
}

__global__ void __launch_bounds__(kD8Threads, kD8CtasPerSm)
    decode_split_fp8_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t d8smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(d8smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kD8Stages * kD8StageBytes);
  uint64_t* empty = full + kD8Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kD8Stages);
  volatile int* never_flag = abort_flag + 1;  // never raised: bounds the drains by time alone

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int lo, hi;
  decode_range(p, p.seqlens[b], lo, hi);
  const int s0 = lo + split * p.chunk;
  const int s1 = min(hi, s0 + p.chunk);
  if (p.nsplit > 1 && s0 >= s1) return;  // empty split: the combine skips it
  const int nkeys = max(0, s1 - s0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kD8Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    *abort_flag = timed_out_before() ? 1 : 0;
    *never_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // after a recorded timeout elsewhere, return at entry: nothing is read or written
  if (*abort_flag) return;
  const int ntiles = (nkeys + kD8TileKeys - 1) / kD8TileKeys;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int row0 = b * p.C + s0;
      int armed = 0;  // tiles whose loads were issued (stage t % kD8Stages)
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % kD8Stages;
        if (t >= kD8Stages) {
          if (!wait_bounded(&empty[st], ((t / kD8Stages) - 1) & 1, abort_flag)) break;
        }
        uint8_t* kb = smem + st * kD8StageBytes;
        uint8_t* vb = kb + kD8KBytes;
        mbar_arrive_expect_tx(&full[st], kD8StageBytes);
        ++armed;
        const int y = row0 + t * kD8TileKeys;
#pragma unroll
        for (int c = 0; c < 3; ++c) tma_load_2d(kb + c * kD8BoxBytes, &tm_k, &full[st], g * 192 + c * 64, y);
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_2d(vb + c * kD8BoxBytes, &tm_v, &full[st], g * 128 + c * 64, y);
      }
      // the CTA never exits with these copies in flight (after a timed-out
      // wait the consumers may have stopped waiting for them)
      for (int s = 0; s < kD8Stages; ++s)
        drain_armed(&full[s], armed > s ? (armed - 1 - s) / kD8Stages + 1 : 0, never_flag);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int r0 = lane >> 2;   // rows (heads) r0 and r0 + 8
    const int t4 = lane & 3;
    const int cq = t4 * 2;      // key pair within an 8-key block (scores, V masks)
    // Q fragments in f16 for the 12 k-steps of 16 dims, in the byte order above:
    // step j, registers {0, 1}: dims 16j+4t, +1 of rows r0 / r0+8; {2, 3}: dims 16j+4t+2, +3.
    uint32_t qa[12][4];
    {
      const int h0 = g * p.G + r0, h1 = g * p.G + r0 + 8;
      const bool v0 = r0 < p.G && MIMO_ROW_OK((long long)b * p.Hq + h0, (long long)p.B * p.Hq);
      const bool v1 = r0 + 8 < p.G && MIMO_ROW_OK((long long)b * p.Hq + h1, (long long)p.B * p.Hq);
      const uint2* q0 = reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.Hq + (v0 ? h0 : 0)) * 192);
      const uint2* q1 = reinterpret_cast<const uint2*>(p.q + ((size_t)b * p.Hq + (v1 ? h1 : 0)) * 192);
#pragma unroll
      for (int j = 0; j < 12; ++j) {
        const int e = (16 * j + 4 * t4) / 4;  // uint2 index: 4 bf16 per load
        const uint2 a = v0 ? __ldg(q0 + e) : make_uint2(0u, 0u);
        const uint2 c = v1 ? __ldg(q1 + e) : make_uint2(0u, 0u);
        qa[j][0] = bf16x2_to_f16x2(a.x);
        qa[j][1] = bf16x2_to_f16x2(c.x);
        qa[j][2] = bf16x2_to_f16x2(a.y);
        qa[j][3] = bf16x2_to_f16x2(c.y);
      }
    }
    const float sl2 = p.scale_log2 * p.k_scale[g];  // code scores -> base-2 logits
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;
    float l0 = 0.f, l1 = 0.f;              // per-thread partial sums (lse)
    float lr0 = 0.f, lr1 = 0.f;            // the same over the rounded P (output normaliser)

    const int kw = warp * 16;
    // ldmatrix row of this lane: matrix m = lane / 8 covers keys kw + 8 (m & 1) + 0..7
    // and the 16-byte column block (m >> 1) of a 32-dim group.
    const int lrow = kw + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int lcol = (lane >> 4) << 4;
    const uint32_t sbase = smem_u32(smem);
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % kD8Stages;
      if (!wait_bounded(&full[st], (t / kD8Stages) & 1, abort_flag)) break;
      const int valid = min(kD8TileKeys, nkeys - t * kD8TileKeys);
      if (kw < valid) {
        const uint32_t kb = sbase + st * kD8StageBytes;
        const uint32_t vb = kb + kD8KBytes;
        // ---- S = Q K^T for keys kw .. kw+15: 6 groups of 32 dims, 4 MMAs each
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int i = 0; i < 6; ++i) {
          const int col = 32 * i + lcol;  // byte column within the 192-byte key row
          uint32_t x0, x1, x2, x3;
          ldsm_x4(kb + (col >> 6) * kD8BoxBytes + sw64_offset(lrow, col & 63), x0, x1, x2, x3);
          uint32_t b[8];
          e4m3x4_to_f16x2x2(x0, b[0], b[1]);
          e4m3x4_to_f16x2x2(x1, b[2], b[3]);
          e4m3x4_to_f16x2x2(x2, b[4], b[5]);
          e4m3x4_to_f16x2x2(x3, b[6], b[7]);
          mma_f16_16816(s[0], qa[2 * i], b[0], b[1]);
          mma_f16_16816(s[1], qa[2 * i], b[2], b[3]);
          mma_f16_16816(s[0], qa[2 * i + 1], b[4], b[5]);
          mma_f16_16816(s[1], qa[2 * i + 1], b[6], b[7]);
        }
        // ---- scale to base 2 and mask keys past the split's end
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = kw + n * 8 + cq + e;
            const bool ok = key < valid;
            s[n][e] = ok ? s[n][e] * sl2 : -INFINITY;
            s[n][2 + e] = ok ? s[n][2 + e] * sl2 : -INFINITY;
            mx0 = fmaxf(mx0, s[n][e]);
            mx1 = fmaxf(mx1, s[n][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float a0 = ex2(m0 - mn0), a1 = ex2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        uint32_t pa[4];
        {
          float p00 = ex2(s[0][0] - mn0), p01 = ex2(s[0][1] - mn0);
          float p02 = ex2(s[0][2] - mn1), p03 = ex2(s[0][3] - mn1);
          float p10 = ex2(s[1][0] - mn0), p11 = ex2(s[1][1] - mn0);
          float p12 = ex2(s[1][2] - mn1), p13 = ex2(s[1][3] - mn1);
          pa[0] = pack_f16(p00, p01);
          pa[1] = pack_f16(p02, p03);
          pa[2] = pack_f16(p10, p11);
          pa[3] = pack_f16(p12, p13);
          l0 = l0 * a0 + ((p00 + p01) + (p10 + p11));
          l1 = l1 * a1 + ((p02 + p03) + (p12 + p13));
          lr0 = lr0 * a0 + ((f16_lo(pa[0]) + f16_hi(pa[0])) + (f16_lo(pa[2]) + f16_hi(pa[2])));
          lr1 = lr1 * a1 + ((f16_lo(pa[1]) + f16_hi(pa[1])) + (f16_lo(pa[3]) + f16_hi(pa[3])));
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
        // ---- O += P V: 4 groups of 32 dims; matrices 0/1 = keys +0..7 / +8..15 of
        // dims +0..15, matrices 2/3 the same keys of dims +16..31.
        const bool partial = (kw + 16 > valid);
        const uint32_t mk0 = (kw + cq < valid ? 0x0000FFFFu : 0u) | (kw + cq + 1 < valid ? 0xFFFF0000u : 0u);
        const uint32_t mk1 = (kw + 8 + cq < valid ? 0x0000FFFFu : 0u) | (kw + 9 + cq < valid ? 0xFFFF0000u : 0u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = 32 * i + lcol;
          uint32_t x0, x1, x2, x3;
          ldsm_x4_t(vb + (col >> 6) * kD8BoxBytes + sw64_offset(lrow, col & 63), x0, x1, x2, x3);
          if (partial) {  // invalid slots may hold anything (NaN codes): zero them
            x0 &= mk0; x1 &= mk1; x2 &= mk0; x3 &= mk1;
          }
          // bytes (k0 d, k0 d+1, k1 d, k1 d+1) -> (k0 d, k1 d, k0 d+1, k1 d+1)
          x0 = prmt(x0, 0u, 0x3120u);
          x1 = prmt(x1, 0u, 0x3120u);
          x2 = prmt(x2, 0u, 0x3120u);
          x3 = prmt(x3, 0u, 0x3120u);
          uint32_t e0[2], e1[2], e2[2], e3[2];  // [0]: dim 2c pairs, [1]: dim 2c+1 pairs
          e4m3x4_to_f16x2x2(x0, e0[0], e0[1]);
          e4m3x4_to_f16x2x2(x1, e1[0], e1[1]);
          e4m3x4_to_f16x2x2(x2, e2[0], e2[1]);
          e4m3x4_to_f16x2x2(x3, e3[0], e3[1]);
          mma_f16_16816(o[4 * i + 0], pa, e0[0], e1[0]);
          mma_f16_16816(o[4 * i + 1], pa, e0[1], e1[1]);
          mma_f16_16816(o[4 * i + 2], pa, e2[0], e3[0]);
          mma_f16_16816(o[4 * i + 3], pa, e2[1], e3[1]);
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
    float* so = reinterpret_cast<float*>(smem);      // [4 warps][16 rows][128]
    float* sm = so + 4 * 16 * 128;                   // [4][16] max
    float* sl = sm + 4 * 16;                         // [4][16] sum
    float* slr = sl + 4 * 16;                        // [4][16] sum of the rounded P
    // o[4i + 2h] holds dims 32i + 16h + {4t, 4t+2} (even MMA), o[4i + 2h + 1]
    // dims 32i + 16h + {4t+1, 4t+3} (odd MMA), for rows r0 (c0, c1) and r0+8 (c2, c3).
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float* ev = o[4 * i + 2 * h];
        const float* od = o[4 * i + 2 * h + 1];
        const int col = 32 * i + 16 * h + 4 * t4;
        *reinterpret_cast<float4*>(so + (warp * 16 + r0) * 128 + col) = make_float4(ev[0], od[0], ev[1], od[1]);
        *reinterpret_cast<float4*>(so + (warp * 16 + r0 + 8) * 128 + col) = make_float4(ev[2], od[2], ev[3], od[3]);
      }
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
    const int tid = threadIdx.x;
    const int row = tid >> 3;
    const int c0 = (tid & 7) * 16;
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
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) a += wgt[w] * so[(w * 16 + row) * 128 + c0 + e];
      acc[e] = a;
    }
    if (row < p.G &&
        (p.nsplit == 1 ? MIMO_ROW_OK((long long)b * p.Hq + g * p.G + row, (long long)p.B * p.Hq)
                       : MIMO_ROW_OK(((long long)b * p.Hkv + g) * p.nsplit + split, (long long)p.B * p.Hkv * p.nsplit))) {
      const int h = g * p.G + row;
      if (p.nsplit == 1) {
        const float sg = p.sinks ? p.sinks[h] * 1.4426950408889634f : -INFINITY;
        const float Mf = fmaxf(M, sg);
        float scl = 0.f, Lf = 0.f, Lrf = 0.f;
        if (Mf != -INFINITY) {
          scl = (M == -INFINITY) ? 0.f : ex2(M - Mf);
          const float ps = (sg == -INFINITY) ? 0.f : ex2(sg - Mf);
          Lf = Ls * scl + ps;
          Lrf = Lrs * scl + ps;
        }
        const float f = (Lrf > 0.f) ? p.v_scale * p.kv_v_scale[g] * scl / Lrf : 0.f;
        const size_t ob = ((size_t)b * p.Hq + h) * 128 + c0;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + ob);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(acc[4 * e] * f, acc[4 * e + 1] * f, acc[4 * e + 2] * f, acc[4 * e + 3] * f);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            uint4 u;
            u.x = pack_bf16(acc[8 * e + 0] * f, acc[8 * e + 1] * f);
            u.y = pack_bf16(acc[8 * e + 2] * f, acc[8 * e + 3] * f);
            u.z = pack_bf16(acc[8 * e + 4] * f, acc[8 * e + 5] * f);
            u.w = pack_bf16(acc[8 * e + 6] * f, acc[8 * e + 7] * f);
            dst[e] = u;
          }
        }
        if (p.lse && (tid & 7) == 0)
          p.lse[(size_t)b * p.Hq + h] = (Lf > 0.f) ? (Mf * 0.6931471805599453f + logf(Lf)) : -INFINITY;
      } else {
        const size_t unit = ((size_t)b * p.Hkv + g) * p.nsplit + split;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (unit * 16 + row) * 128 + c0);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
        if ((tid & 7) == 0) {
          p.ws_ml[(unit * 16 + row) * 4 + 0] = M;
          p.ws_ml[(unit * 16 + row) * 4 + 1] = Ls;
          p.ws_ml[(unit * 16 + row) * 4 + 2] = Lrs;
        }
      }
    }
  }
}

}  // namespace mimo
