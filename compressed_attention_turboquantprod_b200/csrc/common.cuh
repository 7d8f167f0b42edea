// Device helpers shared by the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "tq_internal.h"

namespace tq {

__device__ __forceinline__ float load_f(const void* p, int64_t i, int dtype) {
  if (dtype == TQ_F32) return reinterpret_cast<const float*>(p)[i];
  if (dtype == TQ_F16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ void store_f(void* p, int64_t i, int dtype, float v) {
  if (dtype == TQ_F32) {
    reinterpret_cast<float*>(p)[i] = v;
  } else if (dtype == TQ_F16) {
    reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  } else {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  }
}

__device__ __forceinline__ int dtype_size(int dtype) { return dtype == TQ_F32 ? 4 : 2; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Byte address of field `off`/`size` of absolute compressed token t in region (b, h).
__device__ __forceinline__ uint8_t* field_ptr(uint8_t* base, const Geom& g, int bh, int64_t t,
                                              int off, int size) {
  return base + (int64_t)bh * g.region_bytes + (t / kBlockTokens) * g.block_bytes + off +
         (t % kBlockTokens) * size;
}

// Byte offset, inside a block's value-code field, of 16-bit half x (the codes of
// channels (16/vbits) x ...) of block token tk: the field is 32 token-pair records
// of d*vbits/16 words; half x = gi*H + s (H = g*vbits/16 halves per group) of the
// pair's even token is the low half of word s*(d/g) + gi, the odd token's the high.
__device__ __forceinline__ int vcode_half_off(const Geom& g, int tk, int x) {
  const int H = (g.group * g.vbits) >> 4, NG = g.d / g.group;
  const int word = (x % H) * NG + x / H;
  return (tk >> 1) * 2 * g.f_vcode + 4 * word + 2 * (tk & 1);
}

// Hint: bring the 128-byte line holding p into L2.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Programmatic dependent launch controls (no-ops for an ordinary launch):
// let the next kernel of the stream begin launching, and wait until the
// previous kernel of the stream has completed with its memory visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace tq
