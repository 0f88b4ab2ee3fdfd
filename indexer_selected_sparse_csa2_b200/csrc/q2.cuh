// Staged form of one token's attention query for the tcgen05 attention
// kernel (64 heads x 512 channels): 128 rows, row 2h the fp16 hi part of head
// h's query and row 2h+1 the lo part fp16(q - hi); inside each group of 8
// channels the order is (0, 4, 1, 5, 2, 6, 3, 7).  Channels 0..383 are the
// part that lives in tensor memory (row-major, 192 32-bit words per row: word
// j = the fp16 pair (8g + (j & 3), 8g + (j & 3) + 4), g = j / 4; the 16-byte
// chunk of group g is stored at chunk position g ^ (r & 7) of row r, so that a
// warp reading one chunk of 32 consecutive rows from shared memory touches
// every bank once per 8 rows); channels
// 384..511 the part that lives in shared memory (two K-major 128-byte-swizzled
// blocks of 128 rows x 64 channels).  A decode step can build this once per
// token (prologue) and every split CTA copies it instead of converting q.
#pragma once
#include "sm100.cuh"
#include "rope.cuh"

namespace csa {

constexpr int kQ2TmemWords = 192;                          // per row
constexpr int kQ2TmemBytes = 128 * kQ2TmemWords * 4;       // 96 KB
constexpr int kQ2SmemBytes = 2 * 128 * 128;                // 32 KB
constexpr int kQ2TokenBytes = kQ2TmemBytes + kQ2SmemBytes; // 128 KB

CSA_DEV uint32_t q2_h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Channel held at position p (0..7) of an 8-channel group.
CSA_DEV int perm8(int p) { return (p >> 1) + 4 * (p & 1); }

// fp16 hi / lo parts of 8 channels (a: channels 0-3, c: 4-7) in the staged
// order, as four packed pairs.
CSA_DEV void q_hilo_perm8(float4 a, float4 c, bool lo, uint32_t (&o)[4]) {
  const float f0[4] = {a.x, a.y, a.z, a.w}, f1[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 hi = __floats2half2_rn(f0[k], f1[k]);       // channels k, k + 4
    if (!lo) {
      o[k] = q2_h2u(hi);
    } else {
      const float2 hf = __half22float2(hi);
      o[k] = q2_h2u(__floats2half2_rn(f0[k] - hf.x, f1[k] - hf.y));
    }
  }
}

// One warp stages head h of one token (q_tok: [64][512] fp32) into q2_tok;
// cs_tok: the token's optional [32][2] RoPE table (partial RoPE of channels
// 448..511 before the hi / lo split).
CSA_DEV void encode_q2_head(const float* q_tok, int h, int lane, uint8_t* q2_tok, const float* cs_tok) {
  const float4* src = reinterpret_cast<const float4*>(q_tok + (int64_t)h * 512 + 16 * lane);
  const float4 a0 = src[0], c0 = src[1], a1 = src[2], c1 = src[3];
#pragma unroll
  for (int gg = 0; gg < 2; ++gg) {
    const int g = 2 * lane + gg;                  // channels 8g .. 8g + 7
    float4 a = gg ? a1 : a0, c = gg ? c1 : c0;
    rope_q8(a, c, cs_tok, g);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      uint32_t o[4];
      q_hilo_perm8(a, c, part == 1, o);
      const int r = 2 * h + part;
      uint8_t* dst;
      if (g < 48) {
        dst = q2_tok + ((size_t)r * kQ2TmemWords + 4 * (g ^ (r & 7))) * 4;
      } else {
        const int kb = (g - 48) >> 3, c8 = (g - 48) & 7;
        dst = q2_tok + kQ2TmemBytes + kb * (128 * 128) + sw128_offset_h(r, 8 * c8);
      }
      *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace csa
