// Partial RoPE around the attention, and the output cast.
//
// DeepSeek-V4.1-Flash architecture database: the global layers use partial
// RoPE on the last 64 of the 512 channels of the query and the (cached,
// already rotated) latent, with the inverse rotation applied to the attention
// output; Model techniques map, inference kernels: a fused
// "RoPE-attention-RoPE-cast" kernel.  Channel pairs (448 + 2i, 449 + 2i),
// i = 0..31, are complex numbers multiplied by e^{i theta_i}; the caller
// passes (cos theta_i, sin theta_i) of the query's position, fp32 [32][2] per
// query token.  The output is cast to bf16 (round to nearest even) when asked.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kRopeStart = 448;                  // first rotated channel
constexpr int kRopeGroup0 = kRopeStart / 8;      // first rotated 8-channel group

CSA_DEV float2 rope_fwd(float x, float y, float c, float s) { return make_float2(x * c - y * s, x * s + y * c); }
CSA_DEV float2 rope_inv(float x, float y, float c, float s) { return make_float2(x * c + y * s, y * c - x * s); }

// Rotates the 8 query channels 8g..8g+7 (a: channels 0-3, c: 4-7) forward;
// cs = the token's [32][2] table (nullptr: no RoPE).
CSA_DEV void rope_q8(float4& a, float4& c, const float* cs, int g) {
  if (!cs || g < kRopeGroup0) return;
  const float4 k0 = *reinterpret_cast<const float4*>(cs + 8 * (g - kRopeGroup0));
  const float4 k1 = *reinterpret_cast<const float4*>(cs + 8 * (g - kRopeGroup0) + 4);
  float2 r;
  r = rope_fwd(a.x, a.y, k0.x, k0.y); a.x = r.x; a.y = r.y;
  r = rope_fwd(a.z, a.w, k0.z, k0.w); a.z = r.x; a.w = r.y;
  r = rope_fwd(c.x, c.y, k1.x, k1.y); c.x = r.x; c.y = r.y;
  r = rope_fwd(c.z, c.w, k1.z, k1.w); c.z = r.x; c.w = r.y;
}

// Inverse rotation of 4 output channels d..d+3 (d a multiple of 4).
CSA_DEV float4 rope_out4(float4 v, const float* cs, int d) {
  if (!cs || d < kRopeStart) return v;
  const float4 k = *reinterpret_cast<const float4*>(cs + (d - kRopeStart));
  const float2 r0 = rope_inv(v.x, v.y, k.x, k.y), r1 = rope_inv(v.z, v.w, k.z, k.w);
  return make_float4(r0.x, r0.y, r1.x, r1.y);
}
// ... of 2 output channels d, d+1 (d even).
CSA_DEV float2 rope_out2(float2 v, const float* cs, int d) {
  if (!cs || d < kRopeStart) return v;
  const float2 k = *reinterpret_cast<const float2*>(cs + (d - kRopeStart));
  return rope_inv(v.x, v.y, k.x, k.y);
}

CSA_DEV void store_out4(void* out, bool bf16, int64_t i, float4 v) {
  if (bf16) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + i) = u;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(out) + i) = v;
  }
}
CSA_DEV void store_out2(void* out, bool bf16, int64_t i, float2 v) {
  if (bf16) *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out) + i) = __floats2bfloat162_rn(v.x, v.y);
  else *reinterpret_cast<float2*>(static_cast<float*>(out) + i) = v;
}
CSA_DEV void store_out1(void* out, bool bf16, int64_t i, float v) {
  if (bf16) static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(out)[i] = v;
}

}  // namespace csa
