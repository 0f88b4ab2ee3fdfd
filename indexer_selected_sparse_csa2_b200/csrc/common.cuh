// Shared device helpers of the CSA2 library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <atomic>
#include <utility>

#include "../../include/csa.h"

#define CSA_DEV __device__ __forceinline__

namespace csa {

constexpr int kD = 512;              // latent width (448 nope + 64 rope)
constexpr int kFp4Bytes = 288;       // 256 code bytes + 32 E4M3 scales
constexpr int kFp8Bytes = 528;       // 512 code bytes + 16 UE8M0 exponents
constexpr int kDI = 64;              // indexer head dim
constexpr int kHistBits = 12;        // first-level radix of the Top-K select
constexpr int kHistBins = 1 << kHistBits;
constexpr int kNumSMs = 148;

// ---------------------------------------------------------------- codecs --
// E4M3 ("E4M3FN") encode of two fp32 values, round to nearest even,
// saturating to +-448.  Returns (enc(hi) << 8) | enc(lo).
CSA_DEV uint16_t enc_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// E2M1 encode of two fp32 values (round to nearest even, saturating to +-6).
// Returns (enc(hi) << 4) | enc(lo).
CSA_DEV uint32_t enc_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Exact decodes into fp16x2 (every E2M1 / E4M3 value is an fp16 value).
// Byte b (E2M1 pair): low nibble -> .x, high nibble -> .y.
CSA_DEV __half2 dec_e2m1x2(uint32_t byte) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(r) : "r"(byte));
  return *reinterpret_cast<__half2*>(&r);
}
// Two E4M3 bytes (low byte -> .x, high byte -> .y).
CSA_DEV __half2 dec_e4m3x2(uint32_t two) {
  uint32_t r;
  uint16_t t = (uint16_t)two;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(t));
  return *reinterpret_cast<__half2*>(&r);
}
CSA_DEV float dec_e4m3(uint32_t code) { return __low2float(dec_e4m3x2(code & 0xFF)); }

// Order-preserving 32-bit key of an fp32 value (larger value -> larger key);
// -0 is folded onto +0 first so that equal values have equal keys.
CSA_DEV uint32_t order_key(float v) {
  v = v + 0.0f;
  uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------ misc utils --
CSA_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
CSA_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

CSA_DEV uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
CSA_DEV uint4 ld_v4(const void* p) { return *reinterpret_cast<const uint4*>(p); }

}  // namespace csa

// ------------------------------------------- programmatic dependent launch --
// Every kernel of the library is launched with programmatic stream
// serialization and starts with pdl_enter(): it lets the next kernel on the
// stream be scheduled right away (its CTAs then wait in their own
// pdl_enter()), and waits until the previous kernel on the stream has
// completed and its writes are visible, before touching any memory.  The
// launch latency of each kernel thus overlaps the tail of the one before.
CSA_DEV void pdl_enter() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// The two halves, for a kernel whose prologue reads only memory that no
// kernel of the step writes (caller inputs, or buffers ordered by a full
// stream-event dependency): it triggers at the top, does that prologue while
// the previous kernel still runs, and waits before its first other access.
CSA_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
CSA_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// A kernel attribute (set(): its dynamic shared-memory limit; set_attr(): any
// other), set once per device: cudaFuncSetAttribute applies to the current
// device only, so a process that drives several GPUs must set it on each.
// Thread-safe (a race sets it twice, which is harmless).
class SmemAttrOnce {
 public:
  template <typename... KArgs>
  cudaError_t set(void (*kernel)(KArgs...), size_t bytes) {
    return set_attr(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  }
  template <typename... KArgs>
  cudaError_t set_attr(void (*kernel)(KArgs...), cudaFuncAttribute which, int value) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t)1 << dev : 0;
    if (bit && (done_.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, which, value);
    if (e == cudaSuccess && bit) done_.fetch_or(bit, std::memory_order_acq_rel);
    return e;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// Host-side launch accounting (see csa_launch_count()) and opt-in event
// timing of each launch (see csa_profile_enable()).
namespace csa {
void note_launches(int n);
class ProfScope {
 public:
  ProfScope(cudaStream_t s, const char* name);
  ~ProfScope();
 private:
  cudaStream_t stream_;
  int idx_;
  bool capturing_ = false;
};
}
