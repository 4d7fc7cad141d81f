// Decode step: rotary position embedding of the new token's query and key,
// and the append of its key and value to the cache.
//
// MiMo-V2-Flash model doc: MiMoV2FlashConfig.rope_parameters (rope_theta) and
// MiMoV2FlashModel.forward (position_ids, past_key_values).  The rotation is
// RoFormer's in the rotate-half arrangement: for i < rotary_dim / 2,
// dimensions i and i + rotary_dim / 2 turn by p * theta^(-2 i / rotary_dim)
// at position p = L - 1; dimensions past rotary_dim are unchanged.
//
// One CTA per sequence: the rotary_dim / 2 angles are formed in double
// precision (at p ~ 2^18 an fp32 product p * frequency is off by ~0.02 rad)
// and kept in shared memory as fp32 (cos, sin); the query heads are rotated
// in place, the rotated key and the value are written to the cache slot of
// position p (p mod C for a ring of C slots).
#pragma once

#include "common.cuh"

namespace mimo {

constexpr int kRaThreads = 256;
constexpr int kRaMaxHalf = 96;  // rotary_dim / 2 for head_dim_qk = 192

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
  double theta;
};

__device__ __forceinline__ float2 rope_pair(float x, float y, float2 cs) {
  return make_float2(x * cs.x - y * cs.y, y * cs.x + x * cs.y);
}

__global__ void __launch_bounds__(kRaThreads) rope_append_kernel(const RopeAppendParams p) {
  __shared__ float2 cs[kRaMaxHalf];
  const int b = blockIdx.x;
  const int pos = p.seqlens[b] - 1;
  if (pos < 0 || (!p.ring && pos >= p.C)) {  // the whole CTA takes this branch
    if (threadIdx.x == 0) record_status(1 /* MIMO_ERR_INVALID_ARG */);
    return;
  }
  const int half = p.rotary_dim / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double a = (double)pos * pow(p.theta, -2.0 * i / p.rotary_dim);
    double s, c;
    sincos(a, &s, &c);
    cs[i] = make_float2((float)c, (float)s);
  }
  __syncthreads();
  const int slot = p.ring ? pos % p.C : pos;

  // query heads, in place: one thread per rotation pair
  __nv_bfloat16* q = p.q + (size_t)b * p.Hq * 192;
  for (int w = threadIdx.x; w < p.Hq * half; w += blockDim.x) {
    const int h = w / half, i = w % half;
    __nv_bfloat16* row = q + h * 192;
    const float2 r = rope_pair(__bfloat162float(row[i]), __bfloat162float(row[i + half]), cs[i]);
    row[i] = __float2bfloat16_rn(r.x);
    row[i + half] = __float2bfloat16_rn(r.y);
  }
  // key: rotated into the cache slot (dimensions past rotary_dim copied)
  const __nv_bfloat16* ks = p.k_new + (size_t)b * p.Hkv * 192;
  __nv_bfloat16* kd = p.k_cache + ((size_t)b * p.C + slot) * p.Hkv * 192;
  for (int w = threadIdx.x; w < p.Hkv * 192; w += blockDim.x) {
    const int g = w / 192, d = w % 192;
    const __nv_bfloat16* src = ks + g * 192;
    float val;
    if (d < half) {
      val = rope_pair(__bfloat162float(src[d]), __bfloat162float(src[d + half]), cs[d]).x;
    } else if (d < 2 * half) {
      val = rope_pair(__bfloat162float(src[d - half]), __bfloat162float(src[d]), cs[d - half]).y;
    } else {
      val = __bfloat162float(src[d]);
    }
    kd[g * 192 + d] = __float2bfloat16_rn(val);
  }
  // value: copied into the cache slot
  const __nv_bfloat16* vs = p.v_new + (size_t)b * p.Hkv * 128;
  __nv_bfloat16* vd = p.v_cache + ((size_t)b * p.C + slot) * p.Hkv * 128;
  for (int w = threadIdx.x; w < p.Hkv * 128; w += blockDim.x) vd[w] = vs[w];
}

}  // namespace mimo
