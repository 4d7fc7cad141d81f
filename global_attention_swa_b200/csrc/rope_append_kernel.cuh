// Decode step: rotary position embedding of the new token's query and key,
// and the append of its key and value to the cache.
//
// MiMo-V2-Flash model doc: MiMoV2FlashConfig.rope_parameters (rope_theta) and
// MiMoV2FlashModel.forward (position_ids, past_key_values).  The rotation is
// RoFormer's in the rotate-half arrangement: for i < rotary_dim / 2,
// dimensions i and i + rotary_dim / 2 turn by p * theta^(-2 i / rotary_dim)
// at position p = L - 1; dimensions past rotary_dim are unchanged.
//
// Grid (sequence, group): groups 0 .. ceil(Hq/16)-1 rotate 16 query heads
// each in place, the last group rotates the keys into the cache slot of
// position p (p mod C for a ring of C slots) and copies the values there.
// The frequencies come from the host in double precision; each CTA forms
// p * frequency in double and reduces it modulo 2 pi before the fp32
// sin/cos (at p ~ 2^18 an fp32 product alone would be off by ~0.02 rad).
// With rotary_dim a multiple of 16 a thread turns 8 pairs with 16-byte loads
// and stores; otherwise one pair per thread.
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 6  // site numbers of the checked build

namespace mimo {

constexpr int kRaThreads = 192;
constexpr int kRaMaxHalf = 96;       // rotary_dim / 2 for head_dim_qk = 192
constexpr int kRaHeadsPerCta = 16;

struct RopeAppendParams {
  __nv_bfloat16* q;             // [B, Hq, 192], rotated in place
  const __nv_bfloat16* k_new;   // [B, Hkv, 192], before rotation
  const __nv_bfloat16* v_new;   // [B, Hkv, 128]
  __nv_bfloat16* k_cache;       // [B, C, Hkv, 192]
  __nv_bfloat16* v_cache;       // [B, C, Hkv, 128]
  const int32_t* seqlens;       // [B], the new token included
  int B, C, Hq, Hkv;
  int ring;                     // 1: slot = p mod C
  int rotary_dim;               // even, <= 192
  double inv_freq[kRaMaxHalf];  // theta^(-2 i / rotary_dim)
};

__device__ __forceinline__ float2 rope_pair(float x, float y, float2 cs) {
  return make_float2(x * cs.x - y * cs.y, y * cs.x + x * cs.y);
}

// Rotate the pairs (8j .. 8j+7, half + 8j .. half + 8j + 7) of one 192-dim row.
__device__ __forceinline__ void rope_row8(const __nv_bfloat16* src, __nv_bfloat16* dst, int half, int j,
                                          const float2* cs) {
  const uint4 a = *reinterpret_cast<const uint4*>(src + 8 * j);
  const uint4 b = *reinterpret_cast<const uint4*>(src + half + 8 * j);
  const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
  uint32_t ra[4], rb[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 lo = rope_pair(bf16_lo(av[e]), bf16_lo(bv[e]), cs[8 * j + 2 * e]);
    const float2 hi = rope_pair(bf16_hi(av[e]), bf16_hi(bv[e]), cs[8 * j + 2 * e + 1]);
    ra[e] = pack_bf16(lo.x, hi.x);
    rb[e] = pack_bf16(lo.y, hi.y);
  }
  *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
  *reinterpret_cast<uint4*>(dst + half + 8 * j) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
}

__global__ void __launch_bounds__(kRaThreads) rope_append_kernel(const RopeAppendParams p) {
  __shared__ float2 cs[kRaMaxHalf];
  const int b = blockIdx.x, grp = blockIdx.y;
  const int qgroups = (p.Hq + kRaHeadsPerCta - 1) / kRaHeadsPerCta;
  const int pos = p.seqlens[b] - 1;
  if (pos < 0 || (!p.ring && pos >= p.C)) {  // the whole CTA takes this branch
    if (threadIdx.x == 0 && grp == qgroups) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int half = p.rotary_dim / 2;
  if (threadIdx.x < half) {
    const double a = (double)pos * p.inv_freq[threadIdx.x];
    const double twopi = 6.283185307179586476925286766559;
    const float r = (float)(a - twopi * rint(a / twopi));  // in [-pi, pi]
    float s, c;
    sincosf(r, &s, &c);
    cs[threadIdx.x] = make_float2(c, s);
  }
  __syncthreads();
  const bool vec = (half % 8) == 0;
  const int tasks = vec ? half / 8 : half;  // per row

  if (grp < qgroups) {
    // ---- query heads [16 grp, 16 grp + 16), in place
    const int h0 = grp * kRaHeadsPerCta;
    const int nh = min(kRaHeadsPerCta, p.Hq - h0);
    if (!MIMO_ROW_OK((long long)b * p.Hq + h0 + nh - 1, (long long)p.B * p.Hq)) return;
    __nv_bfloat16* q = p.q + ((size_t)b * p.Hq + h0) * 192;
    for (int w = threadIdx.x; w < nh * tasks; w += blockDim.x) {
      __nv_bfloat16* row = q + (w / tasks) * 192;
      const int j = w % tasks;
      if (vec) {
        rope_row8(row, row, half, j, cs);
      } else {
        const float2 r = rope_pair(__bfloat162float(row[j]), __bfloat162float(row[j + half]), cs[j]);
        row[j] = __float2bfloat16_rn(r.x);
        row[j + half] = __float2bfloat16_rn(r.y);
      }
    }
    return;
  }
  // ---- keys (rotated) and values into the cache slot
  const int slot = p.ring ? pos % p.C : pos;
  if (!MIMO_ROW_OK((long long)b * p.C + slot, (long long)p.B * p.C)) return;
  const __nv_bfloat16* ks = p.k_new + (size_t)b * p.Hkv * 192;
  __nv_bfloat16* kd = p.k_cache + ((size_t)b * p.C + slot) * p.Hkv * 192;
  if (vec) {
    for (int w = threadIdx.x; w < p.Hkv * tasks; w += blockDim.x)
      rope_row8(ks + (w / tasks) * 192, kd + (w / tasks) * 192, half, w % tasks, cs);
  } else {
    for (int w = threadIdx.x; w < p.Hkv * tasks; w += blockDim.x) {
      const int g = w / tasks, j = w % tasks;
      const float2 r = rope_pair(__bfloat162float(ks[g * 192 + j]), __bfloat162float(ks[g * 192 + j + half]), cs[j]);
      kd[g * 192 + j] = __float2bfloat16_rn(r.x);
      kd[g * 192 + j + half] = __float2bfloat16_rn(r.y);
    }
  }
  // dimensions past rotary_dim: copied
  const int tail = 192 - 2 * half;
  for (int w = threadIdx.x; w < p.Hkv * tail; w += blockDim.x) {
    const int g = w / tail, d = 2 * half + w % tail;
    kd[g * 192 + d] = ks[g * 192 + d];
  }
  // values: 16-byte copies (a head row is 256 B)
  const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + (size_t)b * p.Hkv * 128);
  uint4* vd = reinterpret_cast<uint4*>(p.v_cache + ((size_t)b * p.C + slot) * p.Hkv * 128);
  for (int w = threadIdx.x; w < p.Hkv * 16; w += blockDim.x) vd[w] = vs[w];
}

}  // namespace mimo
