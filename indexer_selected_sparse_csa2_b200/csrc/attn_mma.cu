// Sparse MLA attention over gathered FP4 main-KV entries plus the FP8 window.
//
// Multi-head latent attention with one shared latent per position (Model
// techniques map - DeepSeek-V4.1-Flash: "Multi-head latent attention" row and
// num_key_value_heads = 1 in the "Grouped-query attention" row; the
// DeepSeek-V4.1-Flash architecture database stores one shared K=V entry per
// position).  Each query attends to its Top-K selected entries ("Indexer-
// selected sparse attention" row) plus its layer's 128-token sliding window
// ("Sliding-window attention" row); an optional per-head sink logit joins the
// softmax denominator ("Learnable attention sink" row).
//
// Design: all H query heads of one token share every gathered entry, so the
// heads form the M dimension of the contractions and each 288-B entry is read
// and dequantised once per token.  A CTA owns one token and a contiguous
// range of 64-entry tiles (split-K over entries, merged by a log-sum-exp
// combine when a token is split).  Per tile:
//   A  gather + dequantise 64 entries into fp16 shared memory (E2M1 x E4M3
//      and E4M3 values are exact in fp16; window entries are scaled by 2^e in
//      fp32 and rounded to fp16);
//   B  S = Q K^T on tensor cores (mma.sync m16n8k16, fp32 accumulate); Q is
//      held as an fp16 pair hi + lo (lo = fp16(q - hi)), two MMAs per step,
//      so S carries ~22 significant bits of q against the exact fp16 KV;
//   C  online softmax in the exp2 domain, P stored as fp16;
//   D  O += P V on tensor cores, O held in registers (fp32).
// This mma.sync kernel is the alternative path (CSA_ATTN_MMA_SYNC=1); by
// default every head count runs the tcgen05 kernel of attn_tc.cu.
#include <cstdlib>

#include "common.cuh"
#include "attn_tc.cuh"
#include "rope.cuh"

namespace csa {

struct AttnParams {
  int B, n_q, H;
  const float* q;
  const uint8_t* kv;
  int64_t kv_row_stride, kv_batch_stride;
  const int32_t* idx;
  int K;
  const uint8_t* win;
  int64_t win_row_stride, win_batch_stride;
  int n_win;
  float scale_log2;           // softmax_scale * log2(e)
  const float* sink;
  float* out;
  float* lse;
  int n_entries;              // K + n_win
  int tiles_per_split;
  int n_splits;
  float* part_o;              // [B*n_q][n_splits][H][512]
  float* part_ml;             // [B*n_q][n_splits][H][2]
  const float* rope_cs;       // optional [B*n_q][32][2]: partial RoPE of q, inverse on out
  int out_bf16;               // out is bf16
};

constexpr int kAttnThreads = 256;
constexpr int kTileE = 64;                 // entries per tile
constexpr int kQStride = kD + 8;           // halves per shared row (bank-conflict padding)
constexpr int kSStride = kTileE + 4;       // floats per score row
constexpr int kPStride = kTileE + 8;       // halves per P row
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

CSA_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
CSA_DEV void ldsm_x2(uint32_t (&r)[2], const void* p) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(a));
}
CSA_DEV void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
CSA_DEV void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

CSA_DEV uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Channels [128*qq, 128*qq + 128) of an FP4 entry -> fp16 at dst.
// Byte i of the entry holds channels 2i (low nibble) and 2i+1 (high nibble);
// scale byte 256 + k covers channels [16k, 16k + 16).
CSA_DEV void dequant_fp4_quarter(const uint8_t* row, int qq, __half* dst) {
  const uint2 sc = *reinterpret_cast<const uint2*>(row + 256 + 8 * qq);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 c = ld_nc_v4(row + 64 * qq + 16 * v);
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int blk = 2 * v + (k >> 3);
      const uint32_t scode = ((blk < 4 ? sc.x : sc.y) >> (8 * (blk & 3))) & 0xFF;
      const __half2 s2 = __half2half2(__low2half(dec_e4m3x2(scode)));
      const uint32_t byte = (cw[k >> 2] >> (8 * (k & 3))) & 0xFF;
      o[k] = h2_as_u32(__hmul2(dec_e2m1x2(byte), s2));     // exact product
    }
    uint4* d = reinterpret_cast<uint4*>(dst + 32 * v);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
    d[2] = make_uint4(o[8], o[9], o[10], o[11]);
    d[3] = make_uint4(o[12], o[13], o[14], o[15]);
  }
}

// Channels [128*qq, 128*qq + 128) of an FP8 window entry -> fp16 at dst.
// Exponent byte 512 + k (value e + 127) covers channels [32k, 32k + 32).
CSA_DEV void dequant_fp8_quarter(const uint8_t* row, int qq, __half* dst) {
  const uint32_t ew = *reinterpret_cast<const uint32_t*>(row + 512 + 4 * qq);
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint4 c = ld_nc_v4(row + 128 * qq + 16 * v);
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    const int e = (int)((ew >> (8 * (v >> 1))) & 0xFF) - 127;
    const float sc = exp2f((float)e);
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t two = (cw[k >> 1] >> (16 * (k & 1))) & 0xFFFF;
      float2 f = __half22float2(dec_e4m3x2(two));
      o[k] = h2_as_u32(__floats2half2_rn(f.x * sc, f.y * sc));
    }
    uint4* d = reinterpret_cast<uint4*>(dst + 16 * v);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

template <int H>
__global__ void __launch_bounds__(kAttnThreads, 1) sparse_attn_mma_kernel(AttnParams p) {
  pdl_enter();
  constexpr int HB = H / 16;                 // head blocks of 16
  constexpr int EG = 8 / HB;                 // entry groups in phase B
  constexpr int EPW = kTileE / EG;           // entries per warp in phase B
  constexpr int NT_S = EPW / 8;              // n-tiles per warp in phase B
  constexpr int DPW = kD / EG;               // latent channels per warp in phase D
  constexpr int NT_O = DPW / 8;              // n-tiles of O per warp
  constexpr int TPR = kAttnThreads / H;      // softmax threads per head row
  constexpr int EPT = kTileE / TPR;          // entries per softmax thread

  extern __shared__ __align__(16) uint8_t smem[];
  __half* Qs = reinterpret_cast<__half*>(smem);         // hi part of q
  __half* Ql = Qs + H * kQStride;                        // lo part of q
  __half* KVs = Ql + H * kQStride;
  float* Ss = reinterpret_cast<float*>(KVs + kTileE * kQStride);
  __half* Ps = reinterpret_cast<__half*>(Ss + H * kSStride);
  float* m_run = reinterpret_cast<float*>(Ps + H * kPStride);
  float* l_run = m_run + H;
  float* alpha_s = l_run + H;
  int* valid = reinterpret_cast<int*>(alpha_s + H);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int bt = blockIdx.y;                 // b * n_q + t
  const int b = bt / p.n_q, tq = bt - b * p.n_q;
  const int split = blockIdx.x;

  // Q (fp32) -> fp16 shared
  const float* qg = p.q + (int64_t)bt * H * kD;
  for (int i = tid; i < H * kD / 4; i += kAttnThreads) {
    float4 v = reinterpret_cast<const float4*>(qg)[i];
    const int h = (4 * i) / kD, d = (4 * i) % kD;
    if (p.rope_cs && d >= kRopeStart) {
      const float4 k = *reinterpret_cast<const float4*>(p.rope_cs + (int64_t)bt * 64 + (d - kRopeStart));
      const float2 r0 = rope_fwd(v.x, v.y, k.x, k.y), r1 = rope_fwd(v.z, v.w, k.z, k.w);
      v = make_float4(r0.x, r0.y, r1.x, r1.y);
    }
    __half2* dst = reinterpret_cast<__half2*>(Qs + h * kQStride + d);
    __half2* dlo = reinterpret_cast<__half2*>(Ql + h * kQStride + d);
    const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    dst[0] = h01;
    dst[1] = h23;
    dlo[0] = __floats2half2_rn(v.x - f01.x, v.y - f01.y);
    dlo[1] = __floats2half2_rn(v.z - f23.x, v.w - f23.y);
  }
  for (int h = tid; h < H; h += kAttnThreads) { m_run[h] = -INFINITY; l_run[h] = 0.f; }

  float o[NT_O][4];
#pragma unroll
  for (int i = 0; i < NT_O; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  const int hb_b = warp % HB, eg = warp / HB;     // phase B / D roles
  const int32_t* idx = p.idx + (int64_t)bt * p.K;
  const uint8_t* kvb = p.kv + (int64_t)b * p.kv_batch_stride;
  const uint8_t* wb = p.win ? p.win + (int64_t)b * p.win_batch_stride : nullptr;

  const int tile0 = split * p.tiles_per_split;
  const int n_tiles = (p.n_entries + kTileE - 1) / kTileE;
  const int tile1 = min(tile0 + p.tiles_per_split, n_tiles);
  __syncthreads();

  for (int tile = tile0; tile < tile1; ++tile) {
    // ---- A: gather + dequantise (thread -> entry tid/4, channel quarter tid%4)
    {
      const int e = tid >> 2, qq = tid & 3;
      const int j = tile * kTileE + e;
      __half* dst = KVs + e * kQStride + 128 * qq;
      int ok = 0;
      if (j < p.K) {
        const int pos = idx[j];
        if (pos >= 0) {
          dequant_fp4_quarter(kvb + (int64_t)pos * p.kv_row_stride, qq, dst);
          ok = 1;
        }
      } else if (j < p.n_entries) {
        dequant_fp8_quarter(wb + (int64_t)(tq + j - p.K) * p.win_row_stride, qq, dst);
        ok = 1;
      }
      if (!ok) {
        uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int k = 0; k < 16; ++k) d[k] = make_uint4(0, 0, 0, 0);
      }
      if (qq == 0) valid[e] = ok;
    }
    __syncthreads();

    // ---- B: S[h, e] = <Q_h, KV_e> * scale * log2(e)
    {
      float c[NT_S][4];
#pragma unroll
      for (int i = 0; i < NT_S; ++i) c[i][0] = c[i][1] = c[i][2] = c[i][3] = 0.f;
      const __half* qa = Qs + (16 * hb_b + (lane & 15)) * kQStride + 8 * (lane >> 4);
      const __half* qb = qa + H * kQStride;              // same row in the lo part
      const int e0 = eg * EPW;
#pragma unroll 4
      for (int k0 = 0; k0 < kD; k0 += 16) {
        uint32_t a[4], al[4];
        ldsm_x4(a, qa + k0);
        ldsm_x4(al, qb + k0);
        if constexpr (NT_S == 1) {
          uint32_t bb[2];
          ldsm_x2(bb, KVs + (e0 + (lane & 7)) * kQStride + k0 + 8 * ((lane >> 3) & 1));
          mma_f16_16816(c[0], a, bb[0], bb[1]);
          mma_f16_16816(c[0], al, bb[0], bb[1]);
        } else {
#pragma unroll
          for (int nt = 0; nt < NT_S; nt += 2) {
            uint32_t bb[4];
            ldsm_x4(bb, KVs + (e0 + 8 * nt + (lane & 7) + 8 * (lane >> 4)) * kQStride + k0 +
                            8 * ((lane >> 3) & 1));
            mma_f16_16816(c[nt], a, bb[0], bb[1]);
            mma_f16_16816(c[nt + 1], a, bb[2], bb[3]);
            mma_f16_16816(c[nt], al, bb[0], bb[1]);
            mma_f16_16816(c[nt + 1], al, bb[2], bb[3]);
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) {
        const int e = e0 + 8 * nt + 2 * t4;
        const int h = 16 * hb_b + g;
        const bool v0 = valid[e], v1 = valid[e + 1];
        Ss[h * kSStride + e] = v0 ? c[nt][0] * p.scale_log2 : -INFINITY;
        Ss[h * kSStride + e + 1] = v1 ? c[nt][1] * p.scale_log2 : -INFINITY;
        Ss[(h + 8) * kSStride + e] = v0 ? c[nt][2] * p.scale_log2 : -INFINITY;
        Ss[(h + 8) * kSStride + e + 1] = v1 ? c[nt][3] * p.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();

    // ---- C: online softmax per head row
    {
      const int r = tid / TPR, sub = tid % TPR;
      const float* srow = Ss + r * kSStride + sub * EPT;
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < EPT; ++i) mt = fmaxf(mt, srow[i]);
#pragma unroll
      for (int o2 = 1; o2 < TPR; o2 <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o2));
      const float m_old = m_run[r];
      const float m_new = fmaxf(m_old, mt);
      const bool empty = m_new == -INFINITY;
      const float alpha = empty ? 1.f : exp2f(m_old - m_new);
      float ps = 0.f;
      __half* prow = Ps + r * kPStride + sub * EPT;
#pragma unroll
      for (int i = 0; i < EPT; i += 2) {
        const float p0 = empty ? 0.f : exp2f(srow[i] - m_new);
        const float p1 = empty ? 0.f : exp2f(srow[i + 1] - m_new);
        ps += p0 + p1;
        *reinterpret_cast<__half2*>(prow + i) = __floats2half2_rn(p0, p1);
      }
#pragma unroll
      for (int o2 = 1; o2 < TPR; o2 <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      if (sub == 0) {
        l_run[r] = l_run[r] * alpha + ps;
        m_run[r] = m_new;
        alpha_s[r] = alpha;
      }
    }
    __syncthreads();

    // ---- D: O = O * alpha + P V
    {
      const float al0 = alpha_s[16 * hb_b + g], al1 = alpha_s[16 * hb_b + g + 8];
#pragma unroll
      for (int i = 0; i < NT_O; ++i) {
        o[i][0] *= al0; o[i][1] *= al0; o[i][2] *= al1; o[i][3] *= al1;
      }
      const int d0 = eg * DPW;
      const __half* pa = Ps + (16 * hb_b + (lane & 15)) * kPStride + 8 * (lane >> 4);
#pragma unroll
      for (int k0 = 0; k0 < kTileE; k0 += 16) {
        uint32_t a[4];
        ldsm_x4(a, pa + k0);
        const __half* vb = KVs + (k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * kQStride + d0 + 8 * (lane >> 4);
#pragma unroll
        for (int nt = 0; nt < NT_O; nt += 2) {
          uint32_t bb[4];
          ldsm_x4_t(bb, vb + 8 * nt);
          mma_f16_16816(o[nt], a, bb[0], bb[1]);
          mma_f16_16816(o[nt + 1], a, bb[2], bb[3]);
        }
      }
    }
    __syncthreads();
  }

  // ---- epilogue
  const int h0 = 16 * hb_b + g, h1 = h0 + 8;
  const int d0 = eg * DPW;
  if (p.n_splits == 1) {
    // finalise here: fold in the sink, normalise, write out / lse
    float sc0, sc1;
    {
      float m0 = m_run[h0], l0 = l_run[h0], m1 = m_run[h1], l1 = l_run[h1];
      if (p.sink) {
        const float s0 = p.sink[h0] * kLog2e, s1 = p.sink[h1] * kLog2e;
        const float n0 = fmaxf(m0, s0), n1 = fmaxf(m1, s1);
        l0 = (l0 > 0.f ? l0 * exp2f(m0 - n0) : 0.f) + (s0 == -INFINITY ? 0.f : exp2f(s0 - n0));
        l1 = (l1 > 0.f ? l1 * exp2f(m1 - n1) : 0.f) + (s1 == -INFINITY ? 0.f : exp2f(s1 - n1));
        sc0 = l0 > 0.f ? exp2f(m0 - n0) / l0 : 0.f;
        sc1 = l1 > 0.f ? exp2f(m1 - n1) / l1 : 0.f;
        if (m0 == -INFINITY) sc0 = 0.f;
        if (m1 == -INFINITY) sc1 = 0.f;
        m0 = n0; m1 = n1;
      } else {
        sc0 = l0 > 0.f ? 1.f / l0 : 0.f;
        sc1 = l1 > 0.f ? 1.f / l1 : 0.f;
      }
      if (p.lse && eg == 0 && t4 == 0) {
        p.lse[(int64_t)bt * H + h0] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        p.lse[(int64_t)bt * H + h1] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
      }
    }
    const float* cs = p.rope_cs ? p.rope_cs + (int64_t)bt * 64 : nullptr;
    const int64_t o0 = ((int64_t)bt * H + h0) * kD + d0, o1 = ((int64_t)bt * H + h1) * kD + d0;
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) {
      const int d = 8 * nt + 2 * t4;
      store_out2(p.out, p.out_bf16, o0 + d, rope_out2(make_float2(o[nt][0] * sc0, o[nt][1] * sc0), cs, d0 + d));
      store_out2(p.out, p.out_bf16, o1 + d, rope_out2(make_float2(o[nt][2] * sc1, o[nt][3] * sc1), cs, d0 + d));
    }
  } else {
    const int64_t base = ((int64_t)bt * p.n_splits + split) * H;
    float* po0 = p.part_o + (base + h0) * kD + d0;
    float* po1 = p.part_o + (base + h1) * kD + d0;
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) {
      const int d = 8 * nt + 2 * t4;
      *reinterpret_cast<float2*>(po0 + d) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(po1 + d) = make_float2(o[nt][2], o[nt][3]);
    }
    if (eg == 0 && t4 == 0) {
      *reinterpret_cast<float2*>(p.part_ml + (base + h0) * 2) = make_float2(m_run[h0], l_run[h0]);
      *reinterpret_cast<float2*>(p.part_ml + (base + h1) * 2) = make_float2(m_run[h1], l_run[h1]);
    }
  }
}

// Merge the per-split partial results (log-sum-exp combine).  CTA (token,
// head, c) of 128 threads takes channels [128c, 128c + 128) with no shared
// memory and at most 64 registers a thread, so that a combine CTA fits on an
// SM beside one tcgen05 attention CTA (which leaves 8192 registers and no
// shared memory beyond the per-CTA reservation): one layer's combine runs
// while later layers' attention CTAs hold the SMs.  Lane group g = lane / 8
// of each warp takes splits g, g + 4, ... for 8 x 4 channels (its loads in
// flight together), the four groups' sums meet by shuffles.  Every warp
// reduces the splits' (max, sum) partials itself (lane s holds splits s and
// s + 32); split weights 2^(m_s - M) reach the other lanes by shuffles.
constexpr int kCombThreads = 128;
constexpr int kCombChunks = kD / 128;          // channel chunks (grid z)
__global__ void __launch_bounds__(kCombThreads, 8) attn_combine_kernel(AttnParams p) {
  pdl_enter();
  const int bt = blockIdx.x, h = blockIdx.y, H = p.H;
  const int S = p.n_splits;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, g = lane >> 3;
  const int d = 128 * blockIdx.z + 4 * (8 * warp + (lane & 7));
  const float* po = p.part_o + ((int64_t)bt * S * H + h) * kD + d;
  const int64_t sstride = (int64_t)H * kD;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (int64_t)bt * S * H + h;
  constexpr int kR = 8;
  uint4 v[kR];
#pragma unroll
  for (int k = 0; k < kR; ++k) {
    const int s = g + 4 * k;
    v[k] = s < S ? ld_nc_v4(po + s * sstride) : make_uint4(0, 0, 0, 0);
  }
  const float sk = p.sink ? p.sink[h] * kLog2e : -INFINITY;
  const float2 ml0 = lane < S ? ml[(int64_t)lane * H] : make_float2(-INFINITY, 0.f);
  const float2 ml1 = lane + 32 < S ? ml[(int64_t)(lane + 32) * H] : make_float2(-INFINITY, 0.f);
  float M = fmaxf(sk, fmaxf(ml0.x, ml1.x));
  for (int s = lane + 64; s < S; s += 32) M = fmaxf(M, ml[(int64_t)s * H].x);
  M = warp_max(M);
  const float w0 = ml0.x == -INFINITY ? 0.f : exp2f(ml0.x - M);
  const float w1 = ml1.x == -INFINITY ? 0.f : exp2f(ml1.x - M);
  float L = ml0.y * w0 + ml1.y * w1;
  for (int s = lane + 64; s < S; s += 32) {
    const float2 m2 = ml[(int64_t)s * H];
    L += m2.y * (m2.x == -INFINITY ? 0.f : exp2f(m2.x - M));
  }
  L = warp_sum(L);
  if (sk != -INFINITY) L += exp2f(sk - M);
  // weight of split s (s differs between lane groups; every lane shuffles)
  auto weight = [&](int s) -> float {
    const float a = __shfl_sync(0xffffffffu, w0, s & 31);
    const float b = __shfl_sync(0xffffffffu, w1, s & 31);
    if (s < 64) return s < 32 ? a : b;
    if (s >= S) return 0.f;
    const float m = ml[(int64_t)s * H].x;
    return m == -INFINITY ? 0.f : exp2f(m - M);
  };
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0;; s0 += 4 * kR) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int s = s0 + g + 4 * k;
      const float w = weight(s);
      if (s < S) {
        acc.x += w * __uint_as_float(v[k].x); acc.y += w * __uint_as_float(v[k].y);
        acc.z += w * __uint_as_float(v[k].z); acc.w += w * __uint_as_float(v[k].w);
      }
    }
    if (s0 + 4 * kR >= S) break;
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int s = s0 + 4 * kR + g + 4 * k;
      v[k] = s < S ? ld_nc_v4(po + s * sstride) : make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) {
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o); acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o); acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (t == 0 && blockIdx.z == 0 && p.lse) p.lse[(int64_t)bt * H + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  if (g == 0) {
    const float* cs = p.rope_cs ? p.rope_cs + (int64_t)bt * 64 : nullptr;
    store_out4(p.out, p.out_bf16, ((int64_t)bt * H + h) * kD + d,
               rope_out4(make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv), cs, d));
  }
}

template <int H>
static size_t attn_smem_bytes() {
  return (size_t)2 * H * kQStride * 2 + (size_t)kTileE * kQStride * 2 + (size_t)H * kSStride * 4 +
         (size_t)H * kPStride * 2 + (size_t)3 * H * 4 + (size_t)kTileE * 4;
}

struct AttnPlan {
  int n_splits;
  int tiles_per_split;
};

static bool use_tc_attention();

// `share`: how many attention launches of this size are expected to run at
// the same time (concurrent layers of a stack); the SMs are divided among them.
static AttnPlan plan_attn(const csa_attn_args* a, int share) {
  AttnPlan pl;
  const int n_entries = a->K + a->n_win;
  const int n_tiles = (n_entries + kTileE - 1) / kTileE;
  const int64_t tokens = (int64_t)a->B * a->n_q * (share > 1 ? share : 1);
  int want = (int)((kNumSMs + tokens - 1) / tokens);
  // at least two tiles per split on the mma.sync kernel (each split reloads q
  // and writes a partial O); the tcgen05 kernel takes single tiles, its
  // per-split cost is small next to a tile's latency
  const int by_tiles = use_tc_attention() ? n_tiles : (n_tiles + 1) / 2;
  if (want > by_tiles) want = by_tiles;
  if (want < 1) want = 1;
  if (want > n_tiles) want = n_tiles > 0 ? n_tiles : 1;
  pl.tiles_per_split = n_tiles > 0 ? (n_tiles + want - 1) / want : 1;
  pl.n_splits = n_tiles > 0 ? (n_tiles + pl.tiles_per_split - 1) / pl.tiles_per_split : 1;
  return pl;
}

size_t attn_ws_bytes(const csa_attn_args* a, int share) {
  AttnPlan pl = plan_attn(a, share);
  if (pl.n_splits <= 1) return 0;
  const size_t tok = (size_t)a->B * a->n_q;
  return tok * pl.n_splits * a->H * (kD + 2) * 4 + 256;
}

template <int H>
static cudaError_t launch_attn_h(AttnParams& p, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes<H>();
  static SmemAttrOnce attr;
  const cudaError_t ea = attr.set(sparse_attn_mma_kernel<H>, smem);
  if (ea != cudaSuccess) return ea;
  dim3 grid(p.n_splits, p.B * p.n_q);
  {
    ProfScope ps(stream, "sparse_attn_mma");
    launch_k(sparse_attn_mma_kernel<H>, dim3(grid), dim3(kAttnThreads), smem, stream, p);
  }
  note_launches(1);
  if (p.n_splits > 1) {
    ProfScope ps(stream, "attn_combine");
    launch_k(attn_combine_kernel, dim3(p.B * p.n_q, H, kCombChunks), dim3(kCombThreads), 0, stream, p);
    note_launches(1);
  }
  return cudaGetLastError();
}

// CSA_ATTN_MMA_SYNC=1 selects the mma.sync kernel for every head count (both
// kernels are kept: the tcgen05 one is the default).
static bool use_tc_attention() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("CSA_ATTN_MMA_SYNC");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}


// Every head count runs on the tcgen05 kernel (the mma.sync kernel stays as
// the CSA_ATTN_MMA_SYNC=1 alternative).
static cudaError_t launch_attn_tc_any(AttnParams& p, const void* q2, cudaStream_t stream) {
  AttnTcParams t;
  t.q2 = static_cast<const uint8_t*>(q2);
  t.B = p.B; t.n_q = p.n_q; t.H = p.H; t.q = p.q; t.kv = p.kv; t.kv_row_stride = p.kv_row_stride;
  t.kv_batch_stride = p.kv_batch_stride; t.idx = p.idx; t.K = p.K; t.win = p.win;
  t.win_row_stride = p.win_row_stride; t.win_batch_stride = p.win_batch_stride; t.n_win = p.n_win;
  t.scale_log2 = p.scale_log2; t.sink = p.sink; t.out = p.out; t.lse = p.lse; t.n_entries = p.n_entries;
  // the tcgen05 kernel walks 64-entry tiles: same split boundaries
  static_assert(kTileE == 64, "split boundaries must fall on 64-entry tiles");
  t.tiles_per_split = p.tiles_per_split;
  t.n_splits = p.n_splits; t.part_o = p.part_o; t.part_ml = p.part_ml;
  t.rope_cs = p.rope_cs; t.out_bf16 = p.out_bf16;
  cudaError_t e = launch_attn_tc(t, stream);
  if (e != cudaSuccess) return e;
  if (p.n_splits > 1) {
    ProfScope ps(stream, "attn_combine");
    launch_k(attn_combine_kernel, dim3(p.B * p.n_q, p.H, kCombChunks), dim3(kCombThreads), 0, stream, p);
    note_launches(1);
  }
  return cudaGetLastError();
}

// True when these arguments can take q already staged by a layer stack's
// prologue (64 heads on the tcgen05 kernel).
bool attn_tc_path(const csa_attn_args* a) { return a->H == 64 && use_tc_attention(); }

cudaError_t run_sparse_attn(const csa_attn_args* a, void* ws, cudaStream_t stream, const void* q2, int share) {
  AttnPlan pl = plan_attn(a, share);
  AttnParams p{};
  p.B = a->B; p.n_q = a->n_q; p.H = a->H;
  p.q = a->q;
  p.kv = a->kv; p.kv_row_stride = a->kv_row_stride; p.kv_batch_stride = a->kv_batch_stride;
  p.idx = a->idx; p.K = a->K;
  p.win = a->win; p.win_row_stride = a->win_row_stride; p.win_batch_stride = a->win_batch_stride;
  p.n_win = a->n_win;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.sink = a->sink;
  p.out = a->out; p.lse = a->lse;
  p.rope_cs = a->rope_cs; p.out_bf16 = a->out_bf16 != 0;
  p.n_entries = a->K + a->n_win;
  p.tiles_per_split = pl.tiles_per_split;
  p.n_splits = pl.n_splits;
  if (pl.n_splits > 1) {
    const size_t tok = (size_t)a->B * a->n_q;
    p.part_o = static_cast<float*>(ws);
    p.part_ml = p.part_o + tok * pl.n_splits * a->H * kD;
  }
  if (a->H != 16 && a->H != 32 && a->H != 64) return cudaErrorInvalidValue;
  if (use_tc_attention()) return launch_attn_tc_any(p, q2, stream);
  switch (a->H) {
    case 16: return launch_attn_h<16>(p, stream);
    case 32: return launch_attn_h<32>(p, stream);
    default: return launch_attn_h<64>(p, stream);
  }
}

}  // namespace csa
