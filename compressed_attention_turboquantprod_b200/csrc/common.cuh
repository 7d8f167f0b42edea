// Device helpers shared by the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "tq_internal.h"

namespace tq {

// ---------------------------------------------------------------- bounds-checked build
// Built with -DTQ_DEBUG_BOUNDS (libtq_bounds.so), every access whose address is
// computed from cache geometry, token positions or split ranges is first checked
// against the extent of the buffer it belongs to (the cache buffer, a caller's
// array, the workspace).  A failing check records its code in this translation
// unit's flag (first failure wins) and the access is not made: a store goes to a
// sink, a load returns zeros, a bulk copy is not issued (its mbarrier then never
// completes and the consumer's bounded wait gives up).  Nothing traps.  In the
// normal build TQ_CHECKED is the constant true and no check is compiled.
#ifdef TQ_DEBUG_BOUNDS
namespace {
__device__ int g_bounds_code;                        // per translation unit
__device__ __align__(16) unsigned char g_bounds_sink[1024];
}  // namespace
__device__ __forceinline__ bool in_bounds(const void* p, int64_t n, const void* base, int64_t size,
                                          int code) {
  const char* c = static_cast<const char*>(p);
  const char* l = static_cast<const char*>(base);
  if (base != nullptr && c >= l && n >= 0 && c + n <= l + size) return true;
  atomicCAS(&g_bounds_code, 0, code);
  return false;
}
#define TQ_CHECKED(p, n, base, size, code) \
  ::tq::in_bounds((p), (int64_t)(n), (base), (int64_t)(size), (code))
#define TQ_SINK(T) reinterpret_cast<T>(g_bounds_sink)
// Host side: this translation unit's flag, read and cleared (synchronous).
#define TQ_BOUNDS_READER(fn)                                                 \
  int fn() {                                                                 \
    int v = 0, z = 0;                                                        \
    if (cudaMemcpyFromSymbol(&v, g_bounds_code, sizeof(int)) != cudaSuccess) \
      return -1;                                                             \
    if (cudaMemcpyToSymbol(g_bounds_code, &z, sizeof(int)) != cudaSuccess)   \
      return -1;                                                             \
    return v;                                                                \
  }
#else
#define TQ_CHECKED(p, n, base, size, code) ((void)sizeof((size)), true)
#define TQ_SINK(T) static_cast<T>(nullptr)
#define TQ_BOUNDS_READER(fn) \
  int fn() { return 0; }
#endif

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

// In place, the unnormalised Walsh-Hadamard transform y_r = sum_c (-1)^popc(r & c) v_c
// of a d-vector held by one warp (d = 32 NK; element 32 k + lane in v[k]): the
// Sylvester matrix is the Kronecker power of [[1, 1], [1, -1]], so one two-point
// butterfly per index bit gives it (bits 5.. inside a lane's registers, bits 0..4
// across lanes), d log2(d) additions in all.
template <int NK>
__device__ __forceinline__ void warp_fwht(float (&v)[NK], int lane) {
#pragma unroll
  for (int hk = 1; hk < NK; hk <<= 1)
#pragma unroll
    for (int k = 0; k < NK; ++k)
      if (!(k & hk)) {
        const float a = v[k], b = v[k | hk];
        v[k] = a + b;
        v[k | hk] = a - b;
      }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const bool up = (lane & h) != 0;
#pragma unroll
    for (int k = 0; k < NK; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, v[k], h);
      v[k] = up ? o - v[k] : v[k] + o;
    }
  }
}

// Pi u for the structured rotation Pi = H diag(s) / sqrt(d), with pi0 = row 0 of
// Pi (= s / sqrt(d), every entry of Pi being +-pi0[c]): out[r] = scale * (H (pi0 * u))_r,
// one warp, u and out in shared (or global) memory, d in {64, 128, 256}.
__device__ __forceinline__ void warp_hadamard_rotate(const float* pi0, const float* u, float scale,
                                                     float* out, int d, int lane) {
  if (d == 64) {
    float v[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) v[k] = pi0[32 * k + lane] * u[32 * k + lane];
    warp_fwht<2>(v, lane);
#pragma unroll
    for (int k = 0; k < 2; ++k) out[32 * k + lane] = v[k] * scale;
  } else if (d == 128) {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = pi0[32 * k + lane] * u[32 * k + lane];
    warp_fwht<4>(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) out[32 * k + lane] = v[k] * scale;
  } else {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = pi0[32 * k + lane] * u[32 * k + lane];
    warp_fwht<8>(v, lane);
#pragma unroll
    for (int k = 0; k < 8; ++k) out[32 * k + lane] = v[k] * scale;
  }
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
