// Merge of decode results computed over disjoint parts of each sequence's
// keys (context parallelism: a long global-layer cache split across GPUs).
//
// Part r holds the plain-softmax result of its keys without the sink, out_r
// and lse_r = ln sum_{j in r} exp(S_j) (mimo_attn_decode with sinks = NULL).
// With M = max(sigma_h, max_r lse_r) and Z = exp(sigma_h - M) +
// sum_r exp(lse_r - M):  out = v_scale * sum_r exp(lse_r - M) out_r / Z and
// lse = M + ln Z, the decode over all keys with the sink (MiMo-V2-Flash model
// doc, "Key features": learnable attention sink).
//
// One warp per (sequence, query head); lane l owns value columns 4l..4l+3.
#pragma once

#include "common.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 5  // site numbers of the checked build

namespace mimo {

struct DecodeMergeParams {
  const float* part_out;  // [R, B, Hq, 128]
  const float* part_lse;  // [R, B, Hq], natural log, -inf for a part with no keys
  const float* sinks;     // [Hq] or null
  void* out;              // [B, Hq, 128] bf16 or fp32
  float* lse;             // [B, Hq] or null
  int R, B, Hq;
  float v_scale;
  int out_f32;
};

__global__ void __launch_bounds__(256) decode_merge_kernel(const DecodeMergeParams p) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= p.B * p.Hq) return;
  const int b = wid / p.Hq, h = wid % p.Hq;
  const size_t bh = (size_t)b * p.Hq + h;
  const size_t stride = (size_t)p.B * p.Hq;  // between parts
  if (!MIMO_ROW_OK(bh + (size_t)(p.R - 1) * stride, (long long)p.R * stride)) return;
  const float sg = p.sinks ? p.sinks[h] : -INFINITY;
  float M = sg;
  for (int r = 0; r < p.R; ++r) M = fmaxf(M, p.part_lse[r * stride + bh]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Z = 0.f;
  if (M != -INFINITY) {
    Z = (sg == -INFINITY) ? 0.f : expf(sg - M);
    for (int r = 0; r < p.R; ++r) {
      const float x = p.part_lse[r * stride + bh];
      if (x == -INFINITY) continue;  // no keys in this part (its out may be anything)
      const float w = expf(x - M);
      Z += w;
      const float4 o = reinterpret_cast<const float4*>(p.part_out + (r * stride + bh) * 128)[lane];
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
  }
  const float f = (Z > 0.f) ? p.v_scale / Z : 0.f;
  const size_t ob = bh * 128 + lane * 4;
  if (p.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + ob) =
        make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
  } else {
    uint2 u;
    u.x = pack_bf16(acc.x * f, acc.y * f);
    u.y = pack_bf16(acc.z * f, acc.w * f);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + ob) = u;
  }
  if (p.lse && lane == 0) p.lse[bh] = (Z > 0.f) ? (M + logf(Z)) : -INFINITY;
}

}  // namespace mimo
