// Warp-level MMA, mbarrier and bulk-copy helpers shared by the tensor-core
// decode kernels (decode_mma.cu: head dim 128; decode_mma_wide.cu: head dim 256).
#pragma once

#include "common.cuh"

namespace tq {
namespace mmadec {

constexpr int MG = 4;            // query heads per KV head on the tensor-core paths
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kWaitLimit = 1u << 22;

struct MParams {
  Geom g;
  const uint8_t* base;
  int64_t n_comp, n_total;
  int n_ring, Hq;
  float scale_log2;
  float* logits;
  int64_t n_log;
  int splits, bps;
  DecodeWs ws;
  int* err;
  void* out;        // when non-null, the last split of a unit also writes the output
  int64_t early_blk;  // packed blocks [0, early_blk) of every unit are not written by the
                      // grid this kernel is launched programmatically after: their stages
                      // may be requested before the wait for that grid
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ void imma16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void hmma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}


// n consecutive 32-bit words from 16-byte-aligned shared memory, widest loads.
template <int N>
__device__ __forceinline__ void lds_words(const unsigned char* p, uint32_t (&w)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  } else if constexpr (N % 2 == 0) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2*>(p)[i];
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (no transaction count) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// A bulk copy out of the cache buffer [base, base + total); in the bounds-checked
// build a source range outside it is recorded under `code` and not copied.
__device__ __forceinline__ void cache_bulk_load(void* dst, const uint8_t* src, uint32_t bytes,
                                                uint64_t* bar, const uint8_t* base, int64_t total,
                                                int code) {
  if (TQ_CHECKED(src, bytes, base, total, code)) bulk_load(dst, src, bytes, bar);
}

// Packed fp32 pairs (sm_100): one instruction for two IEEE products / fused
// multiply-adds, each rounded exactly as the scalar operation.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&r);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)),
        "l"(*reinterpret_cast<const uint64_t*>(&c)));
  return *reinterpret_cast<const float2*>(&r);
}

// Bounded wait on phase `parity` of an mbarrier for work that takes a while (the
// thread sleeps up to about 0.5 us per poll instead of spinning); false after
// kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity), "r"(500u)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Bounded wait on phase `parity` of an mbarrier; false after kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Named barrier of warp pair `pair` (barrier 1 + pair, 64 threads) that returns the
// OR of `stop` over both warps: the pair's warps take the same decision, so a loop
// that leaves on it keeps every later barrier of the pair matched.
__device__ __forceinline__ bool pair_release(int pair, bool stop) {
  uint32_t any;
  asm volatile(
      "{\n .reg .pred pa, pb;\n setp.ne.u32 pa, %1, 0;\n bar.red.or.pred pb, %2, 64, pa;\n"
      " selp.u32 %0, 1, 0, pb;\n}\n"
      : "=r"(any)
      : "r"((uint32_t)stop), "r"(1 + pair)
      : "memory");
  return any != 0;
}

// The output of a unit from its splits' (m, l, o), run by the CTA of the split that
// finishes last (NT = 32 MG threads, at most 32 splits: a lane per split).  Every
// warp reads the (m, l) of all MG heads, lane s those of split s, and turns them
// into the weights exp2(m_s - M) / L with warp reductions (no shared memory, no
// barrier); thread t sums the channels t + NT c of all heads as sum_s w_s o_s.
// The values of the first eight splits are requested together with (m, l), the
// rest eight splits at a time, so that the merge takes few round trips to L2.
template <int D, int NT>
__device__ __forceinline__ void merge_splits(const MParams& p, int bq0) {
  static_assert(NT == 32 * MG && D % NT == 0, "one warp per head, whole channels per thread");
  constexpr int CPT = D / NT;                 // channels per thread
  constexpr int U = 8;                        // splits per round
  const int tid = threadIdx.x, lane = tid & 31;
  const int S = p.splits;
  const float* po = p.ws.part_o + (int64_t)bq0 * S * D + tid;
  const int64_t hs = (int64_t)S * D;          // stride between heads
  float v[U][MG][CPT];
  auto request = [&](int sp0) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int hh = 0; hh < MG; ++hh)
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          v[u][hh][c] = sp0 + u < S ? __ldcg(po + hh * hs + (int64_t)(sp0 + u) * D + c * NT) : 0.f;
  };
  request(0);
  float w[MG];                                // lane s: the weight of split s, per head
#pragma unroll
  for (int hh = 0; hh < MG; ++hh) {
    float ms = -INFINITY, ls = 0.f;
    if (lane < S) {
      const float* ml = p.ws.part_ml + ((int64_t)(bq0 + hh) * S + lane) * 2;
      ms = __ldcg(ml);
      ls = __ldcg(ml + 1);
    }
    const float M = warp_max(ms);
    const float e = (M == -INFINITY || ms == -INFINITY) ? 0.f : exp2f(ms - M);
    const float L = warp_sum(ls * e);
    w[hh] = e == 0.f ? 0.f : e / L;
  }
  float o[MG][CPT];
#pragma unroll
  for (int hh = 0; hh < MG; ++hh)
#pragma unroll
    for (int c = 0; c < CPT; ++c) o[hh][c] = 0.f;
  for (int sp0 = 0; sp0 < S; sp0 += U) {
    if (sp0 > 0) request(sp0);
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (sp0 + u < S)
#pragma unroll
        for (int hh = 0; hh < MG; ++hh) {
          const float wt = __shfl_sync(0xffffffffu, w[hh], sp0 + u);
#pragma unroll
          for (int c = 0; c < CPT; ++c) o[hh][c] = fmaf(v[u][hh][c], wt, o[hh][c]);
        }
  }
  const int es = p.g.dtype == TQ_F32 ? 4 : 2;
  const int64_t rows = (int64_t)p.g.B * p.Hq;
#pragma unroll
  for (int hh = 0; hh < MG; ++hh)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int64_t e = (int64_t)(bq0 + hh) * D + tid + c * NT;
      if (TQ_CHECKED(static_cast<const char*>(p.out) + e * es, es, p.out, rows * D * es, 117))
        store_f(p.out, e, p.g.dtype, o[hh][c]);
    }
}

// s0 + 2^8 s1 + 2^16 s2 + 2^24 s3 for the four slice sums of a score (each below
// 2^23 in magnitude): the pairs are joined exactly in 32-bit integers (< 2^31),
// then converted once each; the result carries fp32 rounding only.
__device__ __forceinline__ float slices_to_float(int s0, int s1, int s2, int s3) {
  const int lo = s0 + 256 * s1, hi = s2 + 256 * s3;
  return fmaf(65536.f, __int2float_rn(hi), __int2float_rn(lo));
}

// The head-dim-256 kernel (decode_mma_wide.cu).
bool decode_wide_supported(const Geom& g, int G);
cudaError_t launch_partial_wide(const MParams& p, cudaStream_t s);

}  // namespace mmadec
}  // namespace tq
