// Key/value quantisation and append ([TQ] 二 three-stage pipeline, 五
// ProdQuantized, 六 store + ring, 七 value group quantisation).
//
//   keys   rho = ||x||, y = Pi x / rho, idx_j = #{k : beta_k < y_j},
//          e = y - c[idx], ||r|| = rho ||e||, z = rho (T e) with T = S Pi^T,
//          sign bit = [z >= 0]; words LSB-first / little-endian.
//          Pure QJL (b1 = 0): z = S x.
//   values per (token, group): mn, mx, s = (mx - mn)/(2^vb - 1),
//          code = clamp(rint((v - mn)/s)) in IEEE fp32 (__fsub_rn/__fdiv_rn/rintf).
// Three kernels:
//   * head dim 128, m = 128, b1 >= 1, more than 8 tokens: 128-token tiles on the
//     fifth-generation tensor cores (tcgen05 MMAs into tensor memory, one token
//     row per thread in the epilogue; k_quantize_tc);
//   * at most 8 tokens (a decode step's append): a CTA per token (k_quantize_small);
//   * every other shape: 64-token tiles with the contractions as a register-tiled
//     fp32 SGEMM (k_quantize).
#include <cfloat>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "prep_mma.cuh"
#include "tc_common.cuh"

namespace tq {
namespace {

// Tokens per tile of the SGEMM tile quantiser: 64, or 32 where the fp32 tiles of 64
// would leave room for only one CTA per SM (rotated shapes at d >= 128, d = 256).
constexpr int THREADS = 256;
constexpr int NC = 128;       // output columns per GEMM pass
constexpr int KC = 32;        // k-chunk staged in shared memory
constexpr int SBS = NC + 4;   // row stride of the staged B chunk / Z tile

struct QParams {
  // source
  const void* K;
  const void* V;
  int dtype;
  int64_t n, t_first, n_old, n_new;
  bool cache_mode;
  bool fuse_ring;     // cache mode, n_new >= W: the tile kernel also writes the new ring
  const void* ringK;
  const void* ringV;
  // shapes
  int d, b1, m, vbits, group;
  bool do_keys, do_values;
  bool hadamard;      // Pi = H diag(s) / sqrt(d): y = H (Pi[0,:] * x) / rho as a butterfly
  const float* Pi;
  const float* T;
  const float* cent;
  const float* bnd;
  // outputs
  QuantDst arr;
  uint8_t* base;
  Geom g;
};

struct Smem {
  float* X;      // [nt][d+4]
  float* Y;      // [nt][d+4]   (rotated rows; absent when b1 == 0)
  float* B;      // [KC][SBS]
  float* Z;      // [nt][SBS]
  double* rho64; // [nt]
  float* rho;    // [nt]
  float* inv;    // [nt]
  float* cb;     // [16] centroids, [16] boundaries
  float* vs;     // [nt * 16] value scales
  float* vm;     // [nt * 16] value minima
};

__host__ __device__ inline size_t smem_bytes(int d, int nt, int b1) {
  const int sx = d + 4;
  return sizeof(float) * ((b1 > 0 ? 2 : 1) * nt * sx + KC * SBS + nt * SBS) + sizeof(double) * nt +
         sizeof(float) * (2 * nt + 32 + 2 * nt * 16);
}

__device__ Smem carve(unsigned char* raw, int d, int nt, int b1) {
  Smem s;
  const int sx = d + 4;
  double* dp = reinterpret_cast<double*>(raw);
  s.rho64 = dp;
  float* f = reinterpret_cast<float*>(dp + nt);
  s.X = f;
  f += nt * sx;
  s.Y = b1 > 0 ? f : nullptr;
  if (b1 > 0) f += nt * sx;
  s.B = f;
  f += KC * SBS;
  s.Z = f;
  f += nt * SBS;
  s.rho = f;
  f += nt;
  s.inv = f;
  f += nt;
  s.cb = f;
  f += 32;
  s.vs = f;
  f += nt * 16;
  s.vm = f;
  return s;
}

// Element pointer base + index of row i (token t_first + i) of (b, h) in the source.
// (Bounds-checked build: a row outside its buffer reads from the sink.)
__device__ __forceinline__ const void* src_row(const QParams& p, bool values, int bh, int64_t i,
                                               int64_t& elem) {
  const int d = p.d;
  const int es = p.dtype == TQ_F32 ? 4 : 2;
  const void* chunk = values ? p.V : p.K;
  const void* base = chunk;
  [[maybe_unused]] int64_t rows;   // read by the bounds-checked build
  if (!p.cache_mode) {
    elem = i * d;
    rows = p.t_first + p.n;
  } else {
    const int64_t t = p.t_first + i;
    if (t < p.n_old) {
      elem = ((int64_t)bh * p.g.W + t % p.g.W) * d;
      base = values ? p.ringV : p.ringK;
      rows = (int64_t)p.g.B * p.g.Hkv * p.g.W;
    } else {
      elem = ((int64_t)bh * p.n_new + (t - p.n_old)) * d;
      rows = (int64_t)p.g.B * p.g.Hkv * p.n_new;
    }
  }
  if (!TQ_CHECKED(static_cast<const char*>(base) + elem * es, (int64_t)d * es, base,
                  rows * d * es, values ? 402 : 401)) {
    elem = 0;
    return TQ_SINK(const void*);
  }
  return base;
}

// 16-bit half x (codes of channels (16/vbits) x ...) of the value codes of row i:
// token-major in the standalone arrays, token-pair records in the cache.
__device__ __forceinline__ uint16_t* code_half_ptr(const QParams& p, int bh, int64_t i, int x) {
  uint16_t* r;
  if (p.cache_mode) {
    const Geom& g = p.g;
    const int64_t t = p.t_first + i;
    uint8_t* blk = p.base + (int64_t)bh * g.region_bytes + (t / kBlockTokens) * g.block_bytes;
    r = reinterpret_cast<uint16_t*>(blk + g.o_vcode + vcode_half_off(g, (int)(t % kBlockTokens), x));
    if (!TQ_CHECKED(r, 2, p.base, g.total_bytes, 403)) r = TQ_SINK(uint16_t*);
  } else {
    r = reinterpret_cast<uint16_t*>(p.arr.codes + (p.t_first + i) * (p.d * p.vbits / 8)) + x;
    if (!TQ_CHECKED(r, 2, p.arr.codes, (p.t_first + p.n) * (p.d * p.vbits / 8), 404))
      r = TQ_SINK(uint16_t*);
  }
  return r;
}

// Base of row i's value codes and the byte offset of its 16-bit half x from that
// base (code_half_ptr(p, bh, i, x) == code_base(p, bh, i) + code_half_off(p, x)).
__device__ __forceinline__ uint8_t* code_base(const QParams& p, int bh, int64_t i) {
  if (p.cache_mode) {
    const Geom& g = p.g;
    const int64_t t = p.t_first + i;
    uint8_t* blk = p.base + (int64_t)bh * g.region_bytes + (t / kBlockTokens) * g.block_bytes;
    return blk + g.o_vcode + vcode_half_off(g, (int)(t % kBlockTokens), 0);
  }
  return p.arr.codes + (p.t_first + i) * (p.d * p.vbits / 8);
}
__device__ __forceinline__ int code_half_off(const QParams& p, int x) {
  return p.cache_mode ? vcode_half_off(p.g, 0, x) : 2 * x;
}

__device__ __forceinline__ uint8_t* dst_field_raw(const QParams& p, int bh, int64_t i, int which) {
  // which: 0 idx, 1 sign, 2 rho, 3 rnorm, 5 vscale, 6 vmin (value codes: code_half_ptr)
  if (p.cache_mode) {
    const Geom& g = p.g;
    const int64_t t = p.t_first + i;
    switch (which) {
      case 0: return field_ptr(p.base, g, bh, t, g.o_idx, g.f_idx);
      case 1: return field_ptr(p.base, g, bh, t, g.o_sign, g.f_sign);
      case 2: return field_ptr(p.base, g, bh, t, g.o_rho, 4);
      case 3: return field_ptr(p.base, g, bh, t, g.o_rnorm, 4);
      case 5: return field_ptr(p.base, g, bh, t, g.o_vscale, g.f_vmeta);
      default: return field_ptr(p.base, g, bh, t, g.o_vmin, g.f_vmeta);
    }
  }
  const int d = p.d;
  const int64_t ti = p.t_first + i;
  switch (which) {
    case 0: return p.arr.idx + ti * (p.b1 * d / 8);
    case 1: return p.arr.signs + ti * (p.m / 8);
    case 2: return reinterpret_cast<uint8_t*>(p.arr.rho + ti);
    case 3: return reinterpret_cast<uint8_t*>(p.arr.rnorm + ti);
    case 5: return reinterpret_cast<uint8_t*>(p.arr.vscale + ti * (d / p.group));
    default: return reinterpret_cast<uint8_t*>(p.arr.vmin + ti * (d / p.group));
  }
}

// Field `which` of row i (bounds-checked build: the sink when it falls outside
// the cache buffer or the caller's array).
__device__ __forceinline__ uint8_t* dst_field(const QParams& p, int bh, int64_t i, int which) {
  uint8_t* r = dst_field_raw(p, bh, i, which);
#ifdef TQ_DEBUG_BOUNDS
  const int d = p.d;
  const int fsz = which == 0 ? p.b1 * d / 8 : which == 1 ? p.m / 8 : which <= 3 ? 4 : 4 * (d / p.group);
  const void* lo;
  int64_t ext;
  if (p.cache_mode) {
    lo = p.base;
    ext = p.g.total_bytes;
  } else {
    const int64_t rows = p.t_first + p.n;
    lo = which == 0 ? (const void*)p.arr.idx : which == 1 ? (const void*)p.arr.signs
       : which == 2 ? (const void*)p.arr.rho : which == 3 ? (const void*)p.arr.rnorm
       : which == 5 ? (const void*)p.arr.vscale : (const void*)p.arr.vmin;
    ext = rows * fsz;
  }
  if (!TQ_CHECKED(r, fsz, lo, ext, 410 + which)) r = TQ_SINK(uint8_t*);
#endif
  return r;
}

// code = clamp(rint(fl((v - mn) / s)), 0, levels) with fl the IEEE fp32 quotient.
// a * (1/s) is within 3 ulp of fl(a / s) (|quotient| <= 15), so their rints agree
// unless the quotient lies within 1e-5 of a half-integer; only then is the exact
// division taken.  Bit-identical to the plain definition.
__device__ __forceinline__ uint32_t value_code(float v, float mn, float sc, float inv, float levels) {
  if (sc == 0.f) return 0u;
  const float a = __fsub_rn(v, mn);
  const float x = a * inv;
  float r = rintf(x);
  if (fabsf(fabsf(x - r) - 0.5f) < 1e-5f) r = rintf(__fdiv_rn(a, sc));
  r = fminf(fmaxf(r, 0.f), levels);
  return (uint32_t)r;
}

// Four consecutive elements of a row (16-bit types as one 8-byte load).
__device__ __forceinline__ void load4(const void* base, int64_t e, int dtype, float (&o)[4]) {
  if (dtype == TQ_F32) {
    const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + e);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(base) + e);
    const uint32_t w[2] = {u.x, u.y};
    for (int k = 0; k < 2; ++k) {
      if (dtype == TQ_F16) {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
        const float2 f = __half22float2(h);
        o[2 * k] = f.x; o[2 * k + 1] = f.y;
      } else {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
        const float2 f = __bfloat1622float2(h);
        o[2 * k] = f.x; o[2 * k + 1] = f.y;
      }
    }
  }
}

// Load rows [row0, row0+NT) of the key or value source into X (fp32, zero past n):
// a warp per row, the source address computed once per row, 4 elements per lane.
template <int NT>
__device__ void load_tile(const QParams& p, bool values, int bh, int64_t row0, float* X) {
  const int d = p.d, sx = d + 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < NT; r += blockDim.x / 32) {
    const bool valid = row0 + r < p.n;
    int64_t e = 0;
    const void* src = valid ? src_row(p, values, bh, row0 + r, e) : nullptr;
    for (int c = 4 * lane; c < d; c += 128) {
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid) load4(src, e + c, p.dtype, v);
      *reinterpret_cast<float4*>(X + r * sx + c) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// acc[r][c] = sum_k A[RT ty + r][k] * Bg[col0 + tx + 16c][k], k < kdim (RT = NT/16 rows
// per thread); Bg row-major [ncols][kdim], rows past ncols read as zero.
template <int NT>
__device__ void gemm_pass(const float* A, int sa, const float* Bg, int kdim, int col0, int ncols,
                          float* sB, float (&acc)[NT / 16][8]) {
  constexpr int RT = NT / 16;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
  for (int k0 = 0; k0 < kdim; k0 += KC) {
    for (int idx = tid; idx < KC * NC; idx += THREADS) {
      const int kk = idx % KC, c = idx / KC;
      const int col = col0 + c;
      sB[kk * SBS + c] = (col < ncols) ? Bg[(int64_t)col * kdim + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < KC; ++kk) {
      float a[RT], b[8];
#pragma unroll
      for (int r = 0; r < RT; ++r) a[r] = A[(RT * ty + r) * sa + k0 + kk];
#pragma unroll
      for (int c = 0; c < 8; ++c) b[c] = sB[kk * SBS + tx + 16 * c];
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
}

template <int NT>
__device__ void quantize_keys_tile(const QParams& p, const Smem& s, int bh, int64_t row0) {
  constexpr int RT = NT / 16;
  const int d = p.d, sx = d + 4, b1 = p.b1, m = p.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ty = tid / 16, tx = tid % 16;
  load_tile<NT>(p, false, bh, row0, s.X);
  __syncthreads();
  for (int r = warp; r < NT; r += THREADS / 32) {
    double ss = 0.0;
    for (int c = lane; c < d; c += 32) {
      const double x = s.X[r * sx + c];
      ss += x * x;
    }
    ss = warp_sum_d(ss);
    if (lane == 0) {
      const double rho = sqrt(ss);
      s.rho64[r] = rho;
      s.rho[r] = (float)rho;
      s.inv[r] = rho > 0.0 ? (float)(1.0 / rho) : 0.f;
    }
  }
  __syncthreads();
  const float* E = s.X;
  if (b1 > 0) {
    if (p.hadamard) {      // a butterfly per row, one warp each
      for (int r = warp; r < NT; r += THREADS / 32)
        warp_hadamard_rotate(p.Pi, s.X + r * sx, s.inv[r], s.Y + r * sx, d, lane);
    } else {
      for (int col0 = 0; col0 < d; col0 += NC) {
        float acc[RT][8];
        gemm_pass<NT>(s.X, sx, p.Pi, d, col0, d, s.B, acc);
#pragma unroll
        for (int r = 0; r < RT; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int col = col0 + tx + 16 * c;
            if (col < d) s.Y[(RT * ty + r) * sx + col] = acc[r][c] * s.inv[RT * ty + r];
          }
      }
    }
    __syncthreads();
    const int L = 1 << b1;
    for (int r = warp; r < NT; r += THREADS / 32) {
      const bool valid = row0 + r < p.n;
      double se = 0.0;
      uint8_t* idx_dst = valid ? dst_field(p, bh, row0 + r, 0) : nullptr;
      for (int jb = 0; jb < d; jb += 32) {
        const float y = s.Y[r * sx + jb + lane];
        int idx = 0;
        for (int k = 0; k + 1 < L; ++k) idx += (s.cb[16 + k] < y) ? 1 : 0;
        const float e = y - s.cb[idx];
        s.Y[r * sx + jb + lane] = e;
        se += (double)e * (double)e;
        for (int pl = 0; pl < b1; ++pl) {
          const unsigned word = __ballot_sync(0xffffffffu, (idx >> pl) & 1);
          if (lane == 0 && valid)
            *reinterpret_cast<uint32_t*>(idx_dst + pl * (d / 8) + jb / 8) = word;
        }
      }
      se = warp_sum_d(se);
      if (lane == 0 && valid)
        *reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 3)) = (float)(s.rho64[r] * sqrt(se));
    }
    __syncthreads();
    E = s.Y;
  }
  for (int col0 = 0; col0 < m; col0 += NC) {
    float acc[RT][8];
    gemm_pass<NT>(E, sx, p.T, d, col0, m, s.B, acc);
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float z = (b1 > 0) ? acc[r][c] * s.rho[RT * ty + r] : acc[r][c];
        s.Z[(RT * ty + r) * SBS + tx + 16 * c] = z;
      }
    __syncthreads();
    for (int r = warp; r < NT; r += THREADS / 32) {
      const bool valid = row0 + r < p.n;
      uint8_t* sdst = valid ? dst_field(p, bh, row0 + r, 1) : nullptr;
      for (int cb = 0; cb < NC && col0 + cb < m; cb += 32) {
        const unsigned word = __ballot_sync(0xffffffffu, s.Z[r * SBS + cb + lane] >= 0.f);
        if (lane == 0 && valid) *reinterpret_cast<uint32_t*>(sdst + (col0 + cb) / 8) = word;
      }
    }
    __syncthreads();
  }
  for (int r = tid; r < NT; r += THREADS)
    if (row0 + r < p.n) *reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 2)) = s.rho[r];
}

template <int NT>
__device__ void quantize_values_tile(const QParams& p, const Smem& s, int bh, int64_t row0) {
  const int d = p.d, sx = d + 4, g = p.group, ng = d / g, vb = p.vbits;
  const float levels = (float)((1 << vb) - 1);
  const int tid = threadIdx.x;
  load_tile<NT>(p, true, bh, row0, s.X);
  __syncthreads();
  for (int pr = tid; pr < NT * ng; pr += blockDim.x) {
    const int r = pr / ng, gi = pr % ng;
    float mn = FLT_MAX, mx = -FLT_MAX;
    for (int k = 0; k < g; ++k) {
      const float v = s.X[r * sx + gi * g + k];
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
    const float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
    s.vs[pr] = sc;
    s.vm[pr] = mn;
    if (row0 + r < p.n) {
      reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 5))[gi] = sc;
      reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 6))[gi] = mn;
    }
  }
  __syncthreads();
  const int per_word = 32 / vb;
  const int wpr = d / per_word;
  for (int pw = tid; pw < NT * wpr; pw += blockDim.x) {
    const int r = pw / wpr, w = pw % wpr;
    if (row0 + r >= p.n) continue;
    uint32_t word = 0;
    const int gi = (w * per_word) / g;      // a word never straddles two groups (g >= 16)
    const float sc = s.vs[r * ng + gi], mn = s.vm[r * ng + gi];
    const float inv = sc != 0.f ? __frcp_rn(sc) : 0.f;
    for (int k = 0; k < per_word; ++k) {
      const int ch = w * per_word + k;
      word |= value_code(s.X[r * sx + ch], mn, sc, inv, levels) << (k * vb);
    }
    *code_half_ptr(p, bh, row0 + r, 2 * w) = (uint16_t)word;
    *code_half_ptr(p, bh, row0 + r, 2 * w + 1) = (uint16_t)(word >> 16);
  }
  __syncthreads();
}

template <int NT>
__global__ void __launch_bounds__(THREADS) k_quantize(QParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem s = carve(smem_raw, p.d, NT, p.do_keys ? p.b1 : 0);
  const int bh = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * NT;
  if (threadIdx.x < 16) {
    const int L = p.b1 > 0 ? (1 << p.b1) : 0;
    s.cb[threadIdx.x] = (threadIdx.x < L) ? p.cent[threadIdx.x] : 0.f;
    s.cb[16 + threadIdx.x] = (threadIdx.x + 1 < L) ? p.bnd[threadIdx.x] : 0.f;
  }
  __syncthreads();
  if (p.do_keys) quantize_keys_tile<NT>(p, s, bh, row0);
  __syncthreads();
  if (p.do_values) quantize_values_tile<NT>(p, s, bh, row0);
}

__global__ void k_ring_write(Geom g, uint8_t* base, const void* K, const void* V, int64_t n_old,
                             int64_t n_new) {
  // launched programmatically: let the next kernel start, then wait for the
  // previous one (which may still read the ring slots overwritten here)
  pdl_launch_dependents();
  pdl_wait();
  const int bh = blockIdx.x;
  const int es = (g.dtype == TQ_F32) ? 4 : 2;
  const int64_t n_tot = n_old + n_new;
  const int64_t t0 = (n_tot - g.W > n_old) ? n_tot - g.W : n_old;
  const int row_words = g.d * es / 4;
  const int64_t rows = n_tot - t0;
  for (int64_t idx = threadIdx.x; idx < rows * row_words * 2; idx += blockDim.x) {
    const int which = (int)(idx / (rows * row_words));      // 0 = K, 1 = V
    const int64_t rem = idx % (rows * row_words);
    const int64_t t = t0 + rem / row_words;
    const int w = (int)(rem % row_words);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(which ? V : K) +
                          ((int64_t)bh * n_new + (t - n_old)) * row_words;
    uint32_t* dst = reinterpret_cast<uint32_t*>(base + (which ? g.ring_v_off : g.ring_k_off)) +
                    ((int64_t)bh * g.W + t % g.W) * row_words;
    if (TQ_CHECKED(src + w, 4, which ? V : K, (int64_t)g.B * g.Hkv * n_new * row_words * 4, 420) &&
        TQ_CHECKED(dst + w, 4, base, g.total_bytes, 421))
      dst[w] = src[w];
  }
}

// One CTA per token and per half (blockIdx.z = 0: key, 1: value), for launches
// with only a few tokens per (b, kv head) (the decode step appends one): the
// same arithmetic as the 64-token tile.  The key CTA runs its matrix-vector
// products two threads per row (each streams half the row as float4, the vector
// is a shared-memory broadcast) and reduces rho while Pi x is being formed.
constexpr int SMALL_THREADS = 256;

// Half a row of a d x d (or m x d) matrix, d <= 128, held in registers: issued
// early, used later by half_dot.
struct HalfRowRegs {
  float4 w[16];
};
__device__ __forceinline__ void half_row_load(HalfRowRegs& h, const float* rowp, int d, int half) {
  const float4* rp = reinterpret_cast<const float4*>(rowp) + half * (d / 8);
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (i < d / 8) h.w[i] = rp[i];
}
__device__ __forceinline__ float half_dot(const HalfRowRegs& h, const float* v, int d, int half) {
  const float* vp = v + half * (d / 2);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (i < d / 8) {
      const float4 w = h.w[i];
      float& a = (i & 1) ? a1 : a0;
      a = fmaf(w.x, vp[4 * i], a);
      a = fmaf(w.y, vp[4 * i + 1], a);
      a = fmaf(w.z, vp[4 * i + 2], a);
      a = fmaf(w.w, vp[4 * i + 3], a);
    }
  const float a = a0 + a1;
  return a + __shfl_xor_sync(0xffffffffu, a, 1);
}

__device__ __forceinline__ float half_row_dot(const float* rowp, const float* v, int d, int half) {
  const float4* rp = reinterpret_cast<const float4*>(rowp) + half * (d / 8);
  const float* vp = v + half * (d / 2);
  float a = 0.f;
#pragma unroll 8
  for (int i = 0; i < d / 8; ++i) {
    const float4 w = rp[i];
    a = fmaf(w.x, vp[4 * i], a);
    a = fmaf(w.y, vp[4 * i + 1], a);
    a = fmaf(w.z, vp[4 * i + 2], a);
    a = fmaf(w.w, vp[4 * i + 3], a);
  }
  return a + __shfl_xor_sync(0xffffffffu, a, 1);
}

// d elements of `dtype` (a multiple of 16 bytes) from src to dst, 16 bytes a thread.
__device__ __forceinline__ void copy_row16(void* dst, const void* src, int bytes, int tid, int nthreads) {
  for (int i = tid; i < bytes / 16; i += nthreads)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
}

// One token (row) of one (b, kv head): role 0 = key, 1 = value.  When ring_new is
// non-null the token is read from its ring slot and, once it is in shared memory,
// the slot is overwritten with ring_new (the incoming token that takes the slot).
__device__ __forceinline__ void quantize_small_body(const QParams& p, int64_t row, int bh, int role,
                                                    unsigned char* smem_raw, const void* ring_new) {
  const int d = p.d, m = p.m, b1 = p.b1;
  const int es = p.dtype == TQ_F32 ? 4 : 2;
  float* sx = reinterpret_cast<float*>(smem_raw);       // [d]
  float* sy = sx + d;                                    // [d]  Pi x, then e = y - c[idx]
  float* sz = sy + d;                                    // [max(m, 32)]
  __shared__ double s_red[SMALL_THREADS / 32];
  __shared__ float s_cb[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = SMALL_THREADS / 32;
  if (role == 0) {
    if (!p.do_keys) return;
    if (tid < 16) {
      const int L = b1 > 0 ? (1 << b1) : 0;
      s_cb[tid] = (tid < L) ? p.cent[tid] : 0.f;
      s_cb[16 + tid] = (tid + 1 < L) ? p.bnd[tid] : 0.f;
    }
    {
      // this thread's halves of its rows of Pi and T are read after the norm
      const int half = tid & 1;
      for (int j = tid >> 1; j < d; j += SMALL_THREADS / 2)
        if (b1 > 0 && !p.hadamard)
          for (int c = half * (d / 2); c < (half + 1) * (d / 2); c += 32) prefetch_l2(p.Pi + (int64_t)j * d + c);
      for (int a = tid >> 1; a < m; a += SMALL_THREADS / 2)
        for (int c = half * (d / 2); c < (half + 1) * (d / 2); c += 32) prefetch_l2(p.T + (int64_t)a * d + c);
    }
    // d <= 128: this thread's half of Pi row tid / 2 goes out with the key itself
    const bool regs = d <= 128;
    HalfRowRegs hr;
    if (regs && b1 > 0 && !p.hadamard && (tid >> 1) < d)
      half_row_load(hr, p.Pi + (int64_t)(tid >> 1) * d, d, tid & 1);
    int64_t e0;
    const void* src = src_row(p, false, bh, row, e0);
    double ss = 0.0;
    for (int c = tid; c < d; c += SMALL_THREADS) {
      const float v = load_f(src, e0 + c, p.dtype);
      sx[c] = v;
      ss += (double)v * (double)v;
    }
    ss = warp_sum_d(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    if (ring_new &&  // the token is in shared memory: its ring slot takes the new one
        TQ_CHECKED(static_cast<const char*>(src) + e0 * es, d * es, p.base, p.g.total_bytes, 422))
      copy_row16(reinterpret_cast<char*>(const_cast<void*>(src)) + e0 * es, ring_new, d * es, tid,
                 SMALL_THREADS);
    double t = 0.0;
    for (int w = 0; w < NW; ++w) t += s_red[w];
    const double rho64 = sqrt(t);
    const float rho = (float)rho64;
    const float inv = rho64 > 0.0 ? (float)(1.0 / rho64) : 0.f;
    const float* E = sx;
    const int half = tid & 1;
    if (b1 > 0) {
      if (p.hadamard) {       // y = H (Pi[0,:] * x) / rho as a butterfly in warp 0
        if (warp == 0) warp_hadamard_rotate(p.Pi, sx, inv, sy, d, lane);
        if (regs && (tid >> 1) < m) half_row_load(hr, p.T + (int64_t)(tid >> 1) * d, d, half);
      } else if (regs) {
        if ((tid >> 1) < d) {
          const float a = half_dot(hr, sx, d, half);
          if (half == 0) sy[tid >> 1] = a * inv;
        }
        // this thread's half of T row tid / 2, in flight during the codes
        if ((tid >> 1) < m) half_row_load(hr, p.T + (int64_t)(tid >> 1) * d, d, half);
      } else {
        for (int j = tid >> 1; j < d; j += SMALL_THREADS / 2) {
          const float a = half_row_dot(p.Pi + (int64_t)j * d, sx, d, half);
          if (half == 0) sy[j] = a * inv;
        }
      }
      __syncthreads();
      const int L = 1 << b1;
      uint8_t* idx_dst = dst_field(p, bh, row, 0);
      double se = 0.0;
      for (int j = tid; j < d; j += SMALL_THREADS) {
        const float y = sy[j];
        int idx = 0;
        for (int k = 0; k + 1 < L; ++k) idx += (s_cb[16 + k] < y) ? 1 : 0;
        const float e = y - s_cb[idx];
        se += (double)e * (double)e;
        for (int pl = 0; pl < b1; ++pl) {
          const unsigned word = __ballot_sync(0xffffffffu, (idx >> pl) & 1);
          if (lane == 0) *reinterpret_cast<uint32_t*>(idx_dst + pl * (d / 8) + (j - lane) / 8) = word;
        }
        sz[j] = e;                          // staged: sy is still being read by other warps
      }
      se = warp_sum_d(se);
      __syncthreads();
      for (int j = tid; j < d; j += SMALL_THREADS) sy[j] = sz[j];
      if (lane == 0) s_red[warp] = se;
      __syncthreads();
      if (tid == 0) {
        double u = 0.0;
        for (int w = 0; w < NW; ++w) u += s_red[w];
        *reinterpret_cast<float*>(dst_field(p, bh, row, 3)) = (float)(rho64 * sqrt(u));
      }
      E = sy;
    }
    // z = rho T e (or S x), two threads per row; a warp covers 16 rows, so the
    // 32 sign bits of a word come from two warps and are staged in shared memory.
    if (regs && b1 == 0 && (tid >> 1) < m) half_row_load(hr, p.T + (int64_t)(tid >> 1) * d, d, half);
    for (int a = tid >> 1; a < m; a += SMALL_THREADS / 2) {
      const float acc = (regs && a == (tid >> 1)) ? half_dot(hr, E, d, half)
                                                  : half_row_dot(p.T + (int64_t)a * d, E, d, half);
      if (half == 0) sz[a] = (b1 > 0) ? acc * rho : acc;
    }
    __syncthreads();
    uint8_t* sdst = dst_field(p, bh, row, 1);
    for (int ab = warp * 32; ab < m; ab += SMALL_THREADS) {
      const unsigned word = __ballot_sync(0xffffffffu, sz[ab + lane] >= 0.f);
      if (lane == 0) *reinterpret_cast<uint32_t*>(sdst + ab / 8) = word;
    }
    if (tid == 0) *reinterpret_cast<float*>(dst_field(p, bh, row, 2)) = rho;
    return;
  }
  if (!p.do_values) return;
  {
    const int g = p.group, ng = d / g, vb = p.vbits;
    const float levels = (float)((1 << vb) - 1);
    int64_t e0;
    const void* src = src_row(p, true, bh, row, e0);
    for (int c = tid; c < d; c += SMALL_THREADS) sx[c] = load_f(src, e0 + c, p.dtype);
    __syncthreads();
    if (ring_new &&
        TQ_CHECKED(static_cast<const char*>(src) + e0 * es, d * es, p.base, p.g.total_bytes, 423))
      copy_row16(reinterpret_cast<char*>(const_cast<void*>(src)) + e0 * es, ring_new, d * es, tid,
                 SMALL_THREADS);
    float* vs = sz;            // [ng] scales, [ng] minima
    float* vm = sz + 16;
    for (int gi = tid; gi < ng; gi += SMALL_THREADS) {
      float mn = FLT_MAX, mx = -FLT_MAX;
      for (int k = 0; k < g; ++k) {
        const float v = sx[gi * g + k];
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
      const float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
      vs[gi] = sc;
      vm[gi] = mn;
      reinterpret_cast<float*>(dst_field(p, bh, row, 5))[gi] = sc;
      reinterpret_cast<float*>(dst_field(p, bh, row, 6))[gi] = mn;
    }
    __syncthreads();
    const int per_word = 32 / vb, wpr = d / per_word;
    for (int w = tid; w < wpr; w += SMALL_THREADS) {
      uint32_t word = 0;
      const float sc = vs[(w * per_word) / g], mn = vm[(w * per_word) / g];
      const float inv = sc != 0.f ? __frcp_rn(sc) : 0.f;
      for (int k = 0; k < per_word; ++k) {
        const int ch = w * per_word + k;
        word |= value_code(sx[ch], mn, sc, inv, levels) << (k * vb);
      }
      *code_half_ptr(p, bh, row, 2 * w) = (uint16_t)word;
      *code_half_ptr(p, bh, row, 2 * w + 1) = (uint16_t)(word >> 16);
    }
  }
}

__global__ void __launch_bounds__(SMALL_THREADS) k_quantize_small(QParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_launch_dependents();    // the ring write that follows waits for this kernel itself
  quantize_small_body(p, blockIdx.x, blockIdx.y, blockIdx.z, smem_raw, nullptr);
}

// Decode step, first launch: the single-token quantise of the tokens that leave
// the ring (each CTA also writes the incoming token into the ring slot it just
// read), the ring write of incoming tokens whose slot held no token, and the
// query preparation of the tensor-core decode, as one grid of independent CTAs.
struct StepPrep {
  Geom g;
  const void* Q;
  int Hq;
  const float* Pi;
  const float* S;
  const float* cent;
  float scale_log2;
  DecodeWs ws;
};

template <int NV>
__global__ void __launch_bounds__(SMALL_THREADS) k_step_pre(QParams p, int nq_ctas, int nr_ctas,
                                                            StepPrep sp) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_launch_dependents();       // the partial kernel that follows waits for this grid
  const int units = p.g.B * p.g.Hkv;
  const int es = p.dtype == TQ_F32 ? 4 : 2;
  int bid = blockIdx.x;
  if (bid < nq_ctas) {
    const int role = bid & 1, rest = bid >> 1, bh = rest % units;
    const int64_t row = rest / units;                       // token t_first + row leaves the ring
    const int64_t t_new = p.t_first + row + p.g.W;          // the incoming token taking its slot
    const char* chunk = reinterpret_cast<const char*>(role ? p.V : p.K);
    const char* nsrc = chunk + ((int64_t)bh * p.n_new + (t_new - p.n_old)) * p.d * es;
    quantize_small_body(p, row, bh, role, smem_raw, nsrc);
    return;
  }
  bid -= nq_ctas;
  if (bid < nr_ctas) {
    const int bh = bid % units;
    const int64_t j = bid / units;                          // incoming token n_old + j
    const int64_t off = ((int64_t)bh * p.g.W + (p.n_old + j) % p.g.W) * p.d * es;
    const int64_t soff = ((int64_t)bh * p.n_new + j) * p.d * es;
    copy_row16(p.base + p.g.ring_k_off + off, reinterpret_cast<const char*>(p.K) + soff, p.d * es,
               threadIdx.x, SMALL_THREADS);
    copy_row16(p.base + p.g.ring_v_off + off, reinterpret_cast<const char*>(p.V) + soff, p.d * es,
               threadIdx.x, SMALL_THREADS);
    return;
  }
  bid -= nr_ctas;
  mmadec::prep_mma_body<NV>(sp.g, sp.Q, sp.Hq, sp.Pi, sp.S, sp.cent, sp.scale_log2, sp.ws, bid >> 1,
                            bid & 1,
                            smem_raw);
}

// Operands of the tensor-core tile path (head dim 128, b1 > 0, m = 128) are held
// as fp16 hi/lo pairs of v * 2^10 (|lo| <= 2^-11 |hi|); three products hi*hi +
// hi*lo + lo*hi with fp32 accumulation keep about 22 significant bits, well
// inside the 1e-5 band that separates a code or a sign from its decision boundary.
constexpr int QD = 128;             // head dim of this path
constexpr int QM = 128;             // sketch rows of this path
constexpr float kSplit = 1024.f;

// ---------------------------------------------------------------- tcgen05 tiles
// Batched key quantisation on the fifth-generation tensor cores: a persistent
// CTA per SM takes 128-token tiles of one (b, kv head).  Its 16 warps own one
// token row per thread: warp w takes row 32 (w mod 4) + lane (the tensor-memory
// lanes that warp may read) and coordinates 32 (w / 4) .. +31 of it; thread 0
// also issues the MMAs after the barrier that completes their operand.
//   1. rho = ||x|| (fp32 partial sums of 4 squares, float64 total), u = x / rho
//      as f16 hi + lo (x 2^10) into A
//   2. Y = U Pi^T: hi*hi + hi*lo + lo*hi per 16-wide k-step, fp32 in tensor memory;
//      meanwhile the tile's values: per (token, group) mn, s, codes (fp32, IEEE order)
//   3. y, idx_j = #{k : beta_k < y_j}, e = y - c[idx] as hi + lo into A,
//      ||r|| = rho ||e||
//   4. Z = E T^T the same way (T = S Pi^T, so z = rho Z); sign bit [rho Z >= 0]
// Pi and T stay resident as f16 hi + lo in the canonical operand layout.
constexpr int TCM = 128;                   // rows of a tile (MMA M)
constexpr int TC_PARTS = 4;                // 32-coordinate parts of a row
constexpr int TC_THREADS = TCM * TC_PARTS; // 16 warps
constexpr uint32_t TC_COLS = 256;          // tensor-memory columns: the 128 x 128 fp32 tile of the
                                           // hi*hi products, then that of the hi/lo corrections
constexpr int TC_OPB = TCM * QD * 2;       // bytes of one f16 operand (32 KB)
constexpr float kRound = 12582912.f;       // 1.5 * 2^23: x + kRound rounds x (|x| < 2^22) to an integer

__device__ int g_quant_tc_err;             // sticky: a bounded wait gave up

__host__ __device__ inline size_t tc_smem_bytes() {
  return (size_t)6 * TC_OPB + (sizeof(double) * 2 + sizeof(float2)) * TC_PARTS * TCM;
}

// Eight consecutive values (times 2^10) as f16 hi and lo parts, one 16-byte chunk each.
__device__ __forceinline__ void split8(const float (&v)[8], float scale, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 a = mmadec::mul2(make_float2(v[2 * j], v[2 * j + 1]), make_float2(scale, scale));
    const __half2 hh = __floats2half2_rn(a.x, a.y);
    const float2 lf = mmadec::sub2(a, __half22float2(hh));
    const __half2 ll = __floats2half2_rn(lf.x, lf.y);
    h[j] = *reinterpret_cast<const uint32_t*>(&hh);
    l[j] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// The 32 elements of a row segment as raw 16-byte words (issued early, converted
// later): 4 words for 16-bit types, 8 for fp32.  Zeros when !valid.
template <bool F32>
struct RawSeg {
  uint4 w[F32 ? 8 : 4];
};
template <bool F32>
__device__ __forceinline__ void raw_load(RawSeg<F32>& r, const void* base, int64_t e, bool valid) {
  const uint4* src = valid ? reinterpret_cast<const uint4*>(static_cast<const char*>(base) +
                                                            e * (F32 ? 4 : 2))
                           : nullptr;
#pragma unroll
  for (int i = 0; i < (F32 ? 8 : 4); ++i) r.w[i] = valid ? src[i] : make_uint4(0u, 0u, 0u, 0u);
}
template <bool F32>
__device__ __forceinline__ void raw_to_float(const RawSeg<F32>& r, int dtype, float (&o)[32]) {
#pragma unroll
  for (int i = 0; i < (F32 ? 8 : 4); ++i) {
    const uint32_t w[4] = {r.w[i].x, r.w[i].y, r.w[i].z, r.w[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (F32) {
        o[4 * i + k] = __uint_as_float(w[k]);
      } else {
        float2 f;
        if (dtype == TQ_F16) f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        else f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
        o[8 * i + 2 * k] = f.x;
        o[8 * i + 2 * k + 1] = f.y;
      }
    }
  }
}

// code = clamp(rint(fl((v - mn) / s)), 0, levels) as in value_code, with the
// rounding done by adding kRound (exact for 0 <= x < 2^22, ties to even) and
// the integer read from the sum's low mantissa bits.
__device__ __forceinline__ uint32_t value_code_fast(float v, float mn, float sc, float inv, uint32_t levels) {
  if (sc == 0.f) return 0u;
  const float a = __fsub_rn(v, mn);
  const float x = __fmul_rn(a, inv);
  float t = __fadd_rn(x, kRound);
  const float r = __fsub_rn(t, kRound);
  if (fabsf(fabsf(__fsub_rn(x, r)) - 0.5f) < 1e-5f) t = __fadd_rn(rintf(__fdiv_rn(a, sc)), kRound);
  const uint32_t c = __float_as_uint(t) - __float_as_uint(kRound);
  return c < levels ? c : levels;
}

// value_code_fast for two channels sharing mn and inv, in packed fp32 pairs (the
// same IEEE operations, two at a time), without its rare exact-division branch:
// `tie` is set when either product lies within 1e-5 of a half-integer, and the
// caller then recomputes with value_code_fast.
__device__ __forceinline__ void value_code_pair(float v0, float v1, float mn, float inv, uint32_t levels,
                                                uint32_t& c0, uint32_t& c1, bool& tie) {
  const float2 a = mmadec::sub2(make_float2(v0, v1), make_float2(mn, mn));
  const float2 x = mmadec::mul2(a, make_float2(inv, inv));
  const float2 t = mmadec::add2(x, make_float2(kRound, kRound));
  const float2 rr = mmadec::sub2(t, make_float2(kRound, kRound));
  const float2 dd = mmadec::sub2(x, rr);
  // |x - rint(x)| <= 1/2 here, so "within 1e-5 of a half-integer" is one compare
  tie = fabsf(dd.x) > 0.5f - 1e-5f || fabsf(dd.y) > 0.5f - 1e-5f;
  const uint32_t k0 = __float_as_uint(t.x) - __float_as_uint(kRound);
  const uint32_t k1 = __float_as_uint(t.y) - __float_as_uint(kRound);
  c0 = k0 < levels ? k0 : levels;
  c1 = k1 < levels ? k1 : levels;
}

// idx = #{k : beta_k < y} (ascending boundaries beta_0 .. beta_{L-2}) and c[idx], by a
// binary search: bit b1-1 first, each compare choosing between the boundaries of
// the half it selects (selects only: the tables stay in registers).
template <int B1>
__device__ __forceinline__ void code_search(float y, const float* bnd, const float* cen, int& idx,
                                            float& cv) {
  if constexpr (B1 == 1) {
    const bool b0 = bnd[0] < y;
    idx = b0;
    cv = b0 ? cen[1] : cen[0];
  } else if constexpr (B1 == 2) {
    const bool b1 = bnd[1] < y;
    const bool b0 = (b1 ? bnd[2] : bnd[0]) < y;
    idx = 2 * b1 + b0;
    cv = b1 ? (b0 ? cen[3] : cen[2]) : (b0 ? cen[1] : cen[0]);
  } else {
    const bool b2 = bnd[3] < y;
    const bool b1 = (b2 ? bnd[5] : bnd[1]) < y;
    const float t0 = b2 ? (b1 ? bnd[6] : bnd[4]) : (b1 ? bnd[2] : bnd[0]);
    const bool b0 = t0 < y;
    idx = 4 * b2 + 2 * b1 + b0;
    const float lo = b1 ? (b0 ? cen[3] : cen[2]) : (b0 ? cen[1] : cen[0]);
    const float hi = b1 ? (b0 ? cen[7] : cen[6]) : (b0 ? cen[5] : cen[4]);
    cv = b2 ? hi : lo;
  }
}

// The issuing thread: D = A B^T over K = 128 as three products per k-step, the
// hi*hi products into columns 0..127 and the hi*lo + lo*hi corrections into
// 128..255 (the epilogue adds them in fp32: the large partial sums then take one
// accumulation per k-step instead of three).
__device__ __forceinline__ void tc_gemm(uint32_t d_tmem, uint32_t ah, uint32_t al, uint32_t bh,
                                        uint32_t bl) {
  constexpr uint32_t idesc = tc::idesc_f16(TCM, QD);
#pragma unroll
  for (int ks = 0; ks < QD / 16; ++ks) {
    const uint32_t o = 256u * ks;
    tc::mma_f16(d_tmem, tc::smem_desc(ah + o), tc::smem_desc(bh + o), idesc, ks > 0 ? 1u : 0u);
    tc::mma_f16(d_tmem + QD, tc::smem_desc(ah + o), tc::smem_desc(bl + o), idesc, ks > 0 ? 1u : 0u);
    tc::mma_f16(d_tmem + QD, tc::smem_desc(al + o), tc::smem_desc(bh + o), idesc, 1u);
  }
}

// 32 columns of this thread's accumulator row: the hi*hi sums plus the corrections.
__device__ __forceinline__ void tc_ld_sum32(uint32_t taddr, uint32_t (&acc)[32]) {
  tc::tmem_ld32(taddr, acc);
#pragma unroll
  for (int h = 0; h < 2; ++h) {       // the corrections 16 columns at a time (registers)
    uint32_t cor[16];
    tc::tmem_ld16(taddr + QD + 16 * h, cor);
    tc::tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 16; ++c)
      acc[16 * h + c] = __float_as_uint(__uint_as_float(acc[16 * h + c]) + __uint_as_float(cor[c]));
  }
}

// (b, kv head) and first row of tile t of a call: 32-bit division (the host sends a
// call to the tile kernels only when its tiles number below 2^31).
__device__ __forceinline__ int tile_bh(int64_t t, int64_t tiles_per_bh, int64_t& row0) {
  const uint32_t tt = (uint32_t)t, tp = (uint32_t)tiles_per_bh;
  const uint32_t q = tt / tp;
  row0 = (int64_t)(tt - q * tp) * TCM;
  return (int)q;
}

template <int B1, bool F32>
__global__ void __launch_bounds__(TC_THREADS, 1) k_quantize_tc(QParams p, int64_t tiles_per_bh,
                                                              int64_t total_tiles) {
  using mmadec::mbar_init;
  using mmadec::mbar_wait;
  using mmadec::mbar_wait_sleep;
  using mmadec::smem_u32;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_mbar[3];      // Y done, Z done, operand staged
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_hofs[TC_PARTS][8];               // value-code half offsets of each part
  unsigned char* PH = smem_raw;
  unsigned char* PL = PH + TC_OPB;
  unsigned char* TH = PL + TC_OPB;
  unsigned char* TL = TH + TC_OPB;
  unsigned char* AH = TL + TC_OPB;
  unsigned char* AL = AH + TC_OPB;
  double* ssp = reinterpret_cast<double*>(AL + TC_OPB);   // [part][row] partial sums of x^2
  double* sep = ssp + TC_PARTS * TCM;                      // [part][row] partial sums of e^2
  float2* vmm = reinterpret_cast<float2*>(sep + TC_PARTS * TCM);   // [part][row] value min / max
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int L = 1 << B1;

  if (tid == 0) {
    mbar_init(&s_mbar[0], 1);
    mbar_init(&s_mbar[1], 1);
    mbar_init(&s_mbar[2], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  __syncthreads();
  // resident B operands: Pi and T, brought in fp32 by bulk copies (Pi at a
  // 528-byte row stride, so that eight consecutive rows fall in distinct bank
  // groups), then split into f16 hi/lo in the operand layout: row n (output
  // coordinate) over K = 128, a 16-byte chunk (8 consecutive k) per thread and
  // step, eight consecutive rows per eight threads (conflict-free stores)
  const int q = warp & 3, part = warp >> 2;
  const int r = 32 * q + lane;                     // this thread's row of every tile
  const int k0 = 32 * part;                        // and its first coordinate / channel
  const int es = p.dtype == TQ_F32 ? 4 : 2;
  const int g = p.group, vb = p.vbits;
  const uint32_t levels = (1u << vb) - 1u;
  // each part's value-code halves: byte offsets from a row's code base
  if (tid < TC_PARTS * 8) s_hofs[tid >> 3][tid & 7] = code_half_off(p, (32 * (tid >> 3)) * vb / 16 + (tid & 7));
  // this thread's key and value segments of a tile, requested one tile ahead (the
  // first before the operand staging, so that its latency overlaps the staging)
  RawSeg<F32> xr, vr;
  // Launched programmatically (cache appends that write the ring themselves): the
  // kernel before may still run.  Nothing here touches its data except the ring
  // slots (read by a (b, h)'s first tile, which holds the tokens leaving the ring,
  // then rewritten by the same CTA): those tiles wait for it first.
  auto request = [&](int64_t t) {
    bool ok_row = false;
    const void* ks = nullptr;
    const void* vs = nullptr;
    int64_t ek = 0, ev = 0;
    if (t < total_tiles) {
      int64_t tr0;
      const int tbh = tile_bh(t, tiles_per_bh, tr0);
      if (p.cache_mode && p.t_first + tr0 < p.n_old) pdl_wait();     // uniform per tile
      const int64_t trow_i = tr0 + r;
      ok_row = trow_i < p.n;
      if (ok_row) {
        ks = src_row(p, false, tbh, trow_i, ek);
        if (p.do_values) vs = src_row(p, true, tbh, trow_i, ev);
      }
    }
    raw_load(xr, ks, ek + k0, ok_row);
    raw_load(vr, vs, ev + k0, ok_row && p.do_values);
  };
  // the next append's tile kernel may launch (its CTAs take the SMs this grid leaves)
  if (p.fuse_ring) pdl_launch_dependents();
  request(blockIdx.x);

  // Both matrices in one round of bulk copies: Pi's rows into the (not yet used) A
  // area at a 528-byte stride, T's rows unpadded into the Pi operand area; T is
  // split first (into its own operand area), then Pi (into the area T's rows held).
  constexpr int kStage = QD * 4 + 16;
  if (tid == 0) mmadec::mbar_expect_tx(&s_mbar[2], 2 * QD * QD * 4);
  __syncthreads();
  if (tid < 2 * QD) {                                // one row copy per thread
    tc::fence_async_shared();
    if (tid < QD) mmadec::bulk_load(AH + tid * kStage, p.Pi + tid * QD, QD * 4, &s_mbar[2]);
    else mmadec::bulk_load(PH + (tid - QD) * (QD * 4), p.T + (tid - QD) * QD, QD * 4, &s_mbar[2]);
  }
  if (!mbar_wait_sleep(&s_mbar[2], 0u)) s_abort = 1;
  for (int mat = 1; mat >= 0; --mat) {
    // T (unpadded rows): the eight threads of a 16-byte load phase take eight
    // consecutive k chunks (two-way bank conflicts instead of eight-way); the
    // stores stay conflict-free (eight consecutive rows)
    const unsigned char* srcb = mat ? PH : AH;
    const int stride = mat ? QD * 4 : kStage;
    for (int c = tid; c < QD * (QD / 8); c += TC_THREADS) {
      const int n = (c & 7) + 8 * (c >> 7);
      const int kc = mat ? (((c >> 3) + (c & 7)) & 15) : ((c >> 3) & 15);
      const float4 f0 = *reinterpret_cast<const float4*>(srcb + n * stride + 32 * kc);
      const float4 f1 = *reinterpret_cast<const float4*>(srcb + n * stride + 32 * kc + 16);
      const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      uint4 hi, lo;
      split8(v, kSplit, hi, lo);
      const int off = tc::operand_off(n, 8 * kc);
      *reinterpret_cast<uint4*>((mat ? TH : PH) + off) = hi;
      *reinterpret_cast<uint4*>((mat ? TL : PL) + off) = lo;
    }
    __syncthreads();
  }
  float bnd[L - 1], cen[L];
#pragma unroll
  for (int k = 0; k < L; ++k) cen[k] = p.cent[k];
#pragma unroll
  for (int k = 0; k + 1 < L; ++k) bnd[k] = p.bnd[k];
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(&s_tmem), TC_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_async_shared();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t sAH = smem_u32(AH), sAL = smem_u32(AL);
  const uint32_t sPH = smem_u32(PH), sPL = smem_u32(PL), sTH = smem_u32(TH), sTL = smem_u32(TL);

  const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)k0;
  int issued = 0;                                  // thread 0: tiles whose products it issued
  uint32_t it = 0;
  const int64_t tiles_here = *reinterpret_cast<volatile int*>(&s_abort) ? 0 : total_tiles;
  for (int64_t tile = blockIdx.x; tile < tiles_here; tile += gridDim.x, ++it) {
    int64_t row0;
    const int bh = tile_bh(tile, tiles_per_bh, row0);
    const uint32_t ph = it & 1u;
    const int64_t grow = row0 + r;
    const bool valid = grow < p.n;
    {
      // the rows of the tile after next towards L2
      const int64_t nt = tile + 2 * (int64_t)gridDim.x;
      if (nt < tiles_here) {
        int64_t nrow;
        const int nbh = tile_bh(nt, tiles_per_bh, nrow);
        nrow += r;
        if (nrow < p.n) {
          int64_t e0;
          const void* src = src_row(p, false, nbh, nrow, e0);
          prefetch_l2(reinterpret_cast<const char*>(src) + (e0 + k0) * es);
          if (p.do_values) {
            src = src_row(p, true, nbh, nrow, e0);
            prefetch_l2(reinterpret_cast<const char*>(src) + (e0 + k0) * es);
          }
        }
      }
    }
    // ---- 1. rho and U = X / rho
    float inv, rhof;
    double rho64;
    {
      float x[32];
      raw_to_float(xr, p.dtype, x);
      float s8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) s8[j] = 0.f;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 xx = make_float2(x[j], x[j + 1]);
        const float2 sp = mmadec::fma2(xx, xx, make_float2(s8[j & 7], s8[(j + 1) & 7]));
        s8[j & 7] = sp.x;
        s8[(j + 1) & 7] = sp.y;
      }
      double ss = 0.0;
#pragma unroll
      for (int j = 0; j < 8; ++j) ss += (double)s8[j];
      ssp[part * TCM + r] = ss;
      tc::bar_sync(1, TC_THREADS);
      ss = (ssp[r] + ssp[TCM + r]) + (ssp[2 * TCM + r] + ssp[3 * TCM + r]);
      // rho = ss * rsqrt(ss) and 1/rho = rsqrt(ss) (float64)
      const double rs = ss > 0.0 ? rsqrt(ss) : 0.0;
      rho64 = ss * rs;
      rhof = (float)rho64;
      inv = (float)rs;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const float2 u = mmadec::mul2(make_float2(x[8 * c8 + k], x[8 * c8 + k + 1]), make_float2(inv, inv));
          v[k] = u.x;
          v[k + 1] = u.y;
        }
        uint4 hi, lo;
        split8(v, kSplit, hi, lo);
        const int off = tc::operand_off(r, k0 + 8 * c8);
        *reinterpret_cast<uint4*>(AH + off) = hi;
        *reinterpret_cast<uint4*>(AL + off) = lo;
      }
    }
    tc::fence_async_shared();
    tc::fence_before_sync();
    tc::bar_sync(2, TC_THREADS);
    if (tid == 0 && !*reinterpret_cast<volatile int*>(&s_abort)) {
      tc::fence_after_sync();
      tc_gemm(tmem, sAH, sAL, sPH, sPL);
      tc::mma_commit(smem_u32(&s_mbar[0]));
      ++issued;
    }
    // ---- 2. values of this thread's 32 channels, while Y = U Pi^T runs
    if (p.do_values) {
      float v[32];
      raw_to_float(vr, p.dtype, v);
      float mn[2], mx[2];                         // per 16-channel chunk
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        mn[c] = v[16 * c];
        mx[c] = v[16 * c];
#pragma unroll
        for (int k = 1; k < 16; ++k) {
          mn[c] = fminf(mn[c], v[16 * c + k]);
          mx[c] = fmaxf(mx[c], v[16 * c + k]);
        }
      }
      if (g >= 32) {                              // one group covers both chunks
        mn[0] = mn[1] = fminf(mn[0], mn[1]);
        mx[0] = mx[1] = fmaxf(mx[0], mx[1]);
      }
      if (g >= 64) {                              // and the parts of its group
        vmm[part * TCM + r] = make_float2(mn[0], mx[0]);
        tc::bar_sync(1, TC_THREADS);
        const int np = g / 32, p0 = part & ~(np - 1);
        float a = FLT_MAX, b = -FLT_MAX;
        for (int j = 0; j < np; ++j) {
          const float2 m2 = vmm[(p0 + j) * TCM + r];
          a = fminf(a, m2.x);
          b = fmaxf(b, m2.y);
        }
        mn[0] = mn[1] = a;
        mx[0] = mx[1] = b;
      }
      if (valid) {
        float sc[2], iv[2];
        sc[0] = __fdiv_rn(__fsub_rn(mx[0], mn[0]), (float)levels);
        iv[0] = sc[0] != 0.f ? __frcp_rn(sc[0]) : 0.f;
        if (g >= 32) {
          sc[1] = sc[0];
          iv[1] = iv[0];
        } else {
          sc[1] = __fdiv_rn(__fsub_rn(mx[1], mn[1]), (float)levels);
          iv[1] = sc[1] != 0.f ? __frcp_rn(sc[1]) : 0.f;
        }
        // scales / minima: one store per group, by the thread holding its first channel
        float* vsp = reinterpret_cast<float*>(dst_field(p, bh, grow, 5));
        float* vmp = reinterpret_cast<float*>(dst_field(p, bh, grow, 6));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int ch = k0 + 16 * c;
          if (ch % g == 0) {
            vsp[ch / g] = sc[c];
            vmp[ch / g] = mn[c];
          }
        }
        uint8_t* cb = code_base(p, bh, grow);
        // codes of the 32 channels packed as they come (a zero scale has inv = 0, so
        // x = 0 and code 0); near a half-integer (rare) all are redone with the
        // exact division where needed
        const int cpw = 16 / vb;                     // codes per 16-bit half
        uint32_t hw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        bool any_tie = false;
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          bool tie;
          uint32_t c0, c1;
          value_code_pair(v[k], v[k + 1], mn[k >> 4], iv[k >> 4], levels, c0, c1, tie);
          any_tie |= tie && sc[k >> 4] != 0.f;
          if (vb == 2) hw[k >> 3] += (c0 << (2 * (k & 7))) + (c1 << (2 * ((k + 1) & 7)));
          else hw[k >> 2] += (c0 << (4 * (k & 3))) + (c1 << (4 * ((k + 1) & 3)));
        }
        if (any_tie) {
#pragma unroll
          for (int j = 0; j < 8; ++j) hw[j] = 0u;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const uint32_t c = value_code_fast(v[k], mn[k >> 4], sc[k >> 4], iv[k >> 4], levels);
            if (vb == 2) hw[k >> 3] += c << (2 * (k & 7));
            else hw[k >> 2] += c << (4 * (k & 3));
          }
        }
        const int nh = 32 / cpw;
#pragma unroll
        for (int x = 0; x < 8; ++x)
          if (x < nh && TQ_CHECKED(cb + s_hofs[part][x], 2, p.cache_mode ? p.base : p.arr.codes,
                                   p.cache_mode ? p.g.total_bytes
                                                : (p.t_first + p.n) * (p.d * p.vbits / 8), 424))
            *reinterpret_cast<uint16_t*>(cb + s_hofs[part][x]) = (uint16_t)hw[x];
      }
    }
    // the next tile's key and value rows: both register copies are consumed, so the
    // loads have the codes, the second product and the signs to land
    request(tile + gridDim.x);
    // ---- 3. codes, E, ||r||
    bool ok = !*reinterpret_cast<volatile int*>(&s_abort) && mbar_wait_sleep(&s_mbar[0], ph);
    if (!ok) s_abort = 1;
    tc::fence_after_sync();
    uint32_t pw[B1];
    {
      uint32_t acc[32];
      tc_ld_sum32(trow, acc);
#pragma unroll
      for (int pl = 0; pl < B1; ++pl) pw[pl] = 0u;
      float e[32], s8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) s8[j] = 0.f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float2 y2 = mmadec::mul2(make_float2(__uint_as_float(acc[c]), __uint_as_float(acc[c + 1])),
                                       make_float2(1.f / (kSplit * kSplit), 1.f / (kSplit * kSplit)));
        const float yy[2] = {y2.x, y2.y};
        float cv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          // idx = #{k : beta_k < y} by binary search over the ascending boundaries
          // (the same count: the predicate is monotone in k), bits high to low
          int idx;
          code_search<B1>(yy[u], bnd, cen, idx, cv[u]);
#pragma unroll
          for (int pl = 0; pl < B1; ++pl) pw[pl] |= (uint32_t)((idx >> pl) & 1) << (c + u);
        }
        const float2 e2 = mmadec::sub2(y2, make_float2(cv[0], cv[1]));
        e[c] = e2.x;
        e[c + 1] = e2.y;
        const float2 sp = mmadec::fma2(e2, e2, make_float2(s8[c & 7], s8[(c + 1) & 7]));
        s8[c & 7] = sp.x;
        s8[(c + 1) & 7] = sp.y;
      }
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = e[8 * c8 + k];
        uint4 hi, lo;
        split8(v, kSplit, hi, lo);
        const int off = tc::operand_off(r, k0 + 8 * c8);
        *reinterpret_cast<uint4*>(AH + off) = hi;
        *reinterpret_cast<uint4*>(AL + off) = lo;
      }
      double se = 0.0;
#pragma unroll
      for (int j = 0; j < 8; ++j) se += (double)s8[j];
      sep[part * TCM + r] = se;
    }
    tc::fence_async_shared();
    tc::fence_before_sync();
    tc::bar_sync(3, TC_THREADS);
    if (tid == 0 && !*reinterpret_cast<volatile int*>(&s_abort)) {
      tc::fence_after_sync();
      tc_gemm(tmem, sAH, sAL, sTH, sTL);
      tc::mma_commit(smem_u32(&s_mbar[1]));
    }
    if (p.fuse_ring && row0 == 0) {
      // a (b, h)'s first tile: every thread has used its rows (the old ring slots
      // included) before the barrier above, so the new ring (the chunk's last W
      // tokens, token t into slot t mod W) is written now, 16 bytes a thread
      const Geom& gg = p.g;
      const int rb = QD * es / 16;                      // 16-byte words of a row
      for (int i = tid; i < 2 * gg.W * rb; i += TC_THREADS) {
        const int which = i / (gg.W * rb), rem = i % (gg.W * rb), rr = rem / rb, wd = rem % rb;
        const int64_t t = p.n_old + p.n_new - gg.W + rr;            // absolute token
        const uint4* src = reinterpret_cast<const uint4*>(which ? p.V : p.K) +
                           ((int64_t)bh * p.n_new + (t - p.n_old)) * rb + wd;
        uint4* dst = reinterpret_cast<uint4*>(p.base + (which ? gg.ring_v_off : gg.ring_k_off)) +
                     ((int64_t)bh * gg.W + t % gg.W) * rb + wd;
        if (TQ_CHECKED(src, 16, which ? p.V : p.K, (int64_t)gg.B * gg.Hkv * p.n_new * rb * 16, 425) &&
            TQ_CHECKED(dst, 16, p.base, gg.total_bytes, 426))
          *dst = *src;
      }
    }
    const bool write = valid && ok;
    if (write) {
      uint8_t* ip = dst_field(p, bh, grow, 0);
#pragma unroll
      for (int pl = 0; pl < B1; ++pl) *reinterpret_cast<uint32_t*>(ip + pl * (QD / 8) + 4 * part) = pw[pl];
      if (part == 0) {
        const double sev = (sep[r] + sep[TCM + r]) + (sep[2 * TCM + r] + sep[3 * TCM + r]);
        *reinterpret_cast<float*>(dst_field(p, bh, grow, 3)) = (float)(rho64 * sqrt(sev));
        *reinterpret_cast<float*>(dst_field(p, bh, grow, 2)) = rhof;
      }
    }
    // ---- 4. sign bits of z = rho Z
    ok = !*reinterpret_cast<volatile int*>(&s_abort) && mbar_wait_sleep(&s_mbar[1], ph);
    if (!ok) s_abort = 1;
    tc::fence_after_sync();
    {
      uint32_t acc[32];
      tc_ld_sum32(trow, acc);
      // bit = [rho Z >= 0]: for rho > 0 that is [Z >= 0] (a set-on-compare mask per
      // column); a zero rho makes z = 0, every bit 1
      uint32_t pos = 0u;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        uint32_t m;
        asm("set.ge.u32.f32 %0, %1, 0f00000000;" : "=r"(m) : "f"(__uint_as_float(acc[c])));
        pos |= m & (1u << c);
      }
      const uint32_t w = rhof > 0.f ? pos : 0xFFFFFFFFu;
      if (valid && ok) *reinterpret_cast<uint32_t*>(dst_field(p, bh, grow, 1) + 4 * part) = w;
    }
    tc::fence_before_sync();
    tc::bar_sync(4, TC_THREADS);
    if (*reinterpret_cast<volatile int*>(&s_abort)) break;
  }
  if (warp == 0) {
    if (*reinterpret_cast<volatile int*>(&s_abort)) {
      // a wait gave up: let the last products finish (bounded) before freeing
      if (lane == 0) {
        atomicExch(&g_quant_tc_err, 1);
        (void)mbar_wait(&s_mbar[2], 0u);           // the operand copies, if still in flight
        if (issued > 0) {
          (void)mbar_wait(&s_mbar[0], (uint32_t)((issued - 1) & 1));
          (void)mbar_wait(&s_mbar[1], (uint32_t)((issued - 1) & 1));
        }
      }
      __syncwarp();
    }
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TC_COLS);
  }
}

// ---------------------------------------------------------------- tcgen05 tiles, general shapes
// The same pipeline for head dim D in {128, 256}, sketch dim m a multiple of 32 up
// to 512 (the accumulator takes at most the 512 tensor-memory columns) and b1 in
// 0..3 (b1 = 0: pure QJL, z = S x with T = S).  At these shapes Pi and T do not
// fit in shared memory beside the A operand, so they are streamed:
// k_operand_image writes them once per call into a device scratch as f16 hi + lo
// (x kSplit) "pieces" of 128 output rows x 64 K in the canonical K-major layout,
// in the order a tile consumes them (Pi by N-chunk then K-chunk, then T the same
// way); a tensor warp copies the pieces into shared-memory stages (bulk copies
// completing on an mbarrier), issues each piece's MMAs (three hi/lo products per
// 16-wide k-step) and commits them to the barrier that frees the stage, running
// ahead into the next tile while the epilogue works.  The 16 epilogue warps hold
// one token row per thread as in k_quantize_tc, D/4 coordinates (D/128 words of
// 32) per thread:
//   U -> A;  [b1 > 0: Y = U Pi^T; codes, E -> A];  Z = A T^T;  sign bits.
constexpr int TG_EPI = 512;                   // epilogue threads (16 warps)
constexpr int TG_THREADS = TG_EPI + 32;       // and the tensor warp
constexpr int TG_KC = 64;                     // K of one operand piece
constexpr int TG_PIECE = 128 * TG_KC * 4;     // bytes of a full piece (f16 hi + lo)
constexpr int TG_OPS = 192 * 1024;            // shared memory of A and the stages

__host__ __device__ constexpr int tg_stages(int D) { return (TG_OPS - 512 * D) / TG_PIECE; }
__host__ __device__ inline size_t tg_smem_bytes() {
  return (size_t)TG_OPS + (sizeof(double) * 2 + sizeof(float2)) * TC_PARTS * TCM;
}
// Bytes of the operand image: Pi (b1 > 0) and T, 4 bytes (hi + lo) per element.
__host__ __device__ inline size_t tg_image_bytes(int D, int b1, int m) {
  return (size_t)4 * D * ((b1 > 0 ? D : 0) + m);
}
// With b1 > 0 the hi*hi products accumulate apart from the hi*lo + lo*hi
// corrections (two accumulators, summed in fp32 by the epilogue), so that the
// large partial sums take one accumulation per k-step instead of three: the
// residual e = y - c[idx] is an order of magnitude below y, and its sketch
// z = T e carries y's absolute error times sqrt(d), so y needs close to fp32
// accuracy (measured at d = 256: sign decisions within 7e-6 of the rms |z| with
// one accumulator, against 1.3e-6 for the fp32 CUDA-core product).  Pure QJL
// (z = S u, no residual) keeps one.
__host__ __device__ inline bool tg_split_acc(int D, int b1, int m) {
  return b1 > 0 && 2 * (D > m ? D : m) <= 512;
}
// Tensor-memory columns: a power of two >= max(D (b1 > 0), m, 32), twice that
// with split accumulators (the corrections at + half).
__host__ __device__ inline uint32_t tg_tmem_cols(int D, int b1, int m) {
  const int need = (b1 > 0 && D > m) ? D : m;
  uint32_t c = 32;
  while ((int)c < need) c <<= 1;
  return tg_split_acc(D, b1, m) ? 2 * c : c;
}

// Piece c of a tile's sequence (nY = pieces of Pi): its byte offset in the image,
// rows (the MMA's N), first accumulator column and K chunk.  Every N-chunk but the
// last of T has 128 rows; a piece of r rows takes 256 r bytes.
struct TgPiece {
  uint32_t off;
  int nr, dcol, kc;
};
__host__ __device__ inline TgPiece tg_piece(int c, int D, int m, int nY) {
  const int kpn = D / TG_KC;
  TgPiece pc;
  if (c < nY) {
    pc.kc = c % kpn;
    pc.nr = 128;
    pc.dcol = 128 * (c / kpn);
    pc.off = (uint32_t)c * TG_PIECE;
  } else {
    const int j = c - nY, nc = j / kpn;
    pc.kc = j % kpn;
    pc.nr = m - 128 * nc < 128 ? m - 128 * nc : 128;
    pc.dcol = 128 * nc;
    pc.off = (uint32_t)(nY + nc * kpn) * TG_PIECE + (uint32_t)(pc.kc * pc.nr * 256);
  }
  return pc;
}

// One thread per 8 consecutive K of a row of Pi (b1 > 0) or T: f16 hi + lo
// (x kSplit), hi at the row's place in its piece, lo r * 128 bytes further.
__global__ void k_operand_image(const float* Pi, const float* T, int D, int b1, int m,
                                uint8_t* img, int64_t img_bytes) {
  pdl_launch_dependents();     // the quantiser may start its own prologue
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int k8 = D / 8, rowsY = b1 > 0 ? D : 0;
  if (i >= (int64_t)(rowsY + m) * k8) return;
  const int row = (int)(i / k8), k = 8 * (int)(i % k8);
  const bool isY = row < rowsY;
  const int n = isY ? row : row - rowsY;
  const float4* src = reinterpret_cast<const float4*>((isY ? Pi : T) + (int64_t)n * D + k);
  const float4 f0 = src[0], f1 = src[1];
  const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
  uint4 hi, lo;
  split8(v, kSplit, hi, lo);
  const int kpn = D / TG_KC, nY = rowsY > 0 ? (D / 128) * kpn : 0;
  const int rl = n % 128, kl = k % TG_KC;
  const TgPiece pc = tg_piece((isY ? 0 : nY) + (n / 128) * kpn + k / TG_KC, D, m, nY);
  const uint32_t o = pc.off + (uint32_t)((((rl >> 3) * 8) + (kl >> 3)) * 128 + (rl & 7) * 16);
  if (TQ_CHECKED(img + o, 16, img, img_bytes, 431)) *reinterpret_cast<uint4*>(img + o) = hi;
  if (TQ_CHECKED(img + o + pc.nr * 128, 16, img, img_bytes, 432))
    *reinterpret_cast<uint4*>(img + o + pc.nr * 128) = lo;
}

template <int D, int B1, bool F32>
__global__ void __launch_bounds__(TG_THREADS, 1) k_quantize_tcg(QParams p, const uint8_t* img,
                                                               int64_t img_bytes, int64_t tiles_per_bh,
                                                               int64_t total_tiles) {
  using mmadec::mbar_init;
  using mmadec::mbar_wait;
  using mmadec::mbar_wait_sleep;
  using mmadec::smem_u32;
  constexpr int NW = D / 128;                  // 32-coordinate words per thread
  constexpr int NS = tg_stages(D);             // piece stages
  constexpr int KPN = D / TG_KC;               // pieces per N-chunk
  constexpr int NY = B1 > 0 ? (D / 128) * KPN : 0;
  constexpr int L = B1 > 0 ? 1 << B1 : 2;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_full[NS], s_empty[NS];
  __shared__ __align__(8) uint64_t s_aready, s_ydone, s_zdone, s_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_hofs[TC_PARTS][16];         // value-code half offsets of each part
  unsigned char* AH = smem_raw;
  unsigned char* AL = AH + 256 * D;
  unsigned char* ST = AL + 256 * D;            // [NS][TG_PIECE]
  double* ssp = reinterpret_cast<double*>(smem_raw + TG_OPS);      // [part][row] sums of x^2
  double* sep = ssp + TC_PARTS * TCM;                                // [part][row] sums of e^2
  float2* vmm = reinterpret_cast<float2*>(sep + TC_PARTS * TCM);    // [part][row] value min / max
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m = p.m;
  const int nC = NY + ((m + 127) / 128) * KPN;
  const uint32_t tcols = tg_tmem_cols(D, B1, m);
  const bool split = tg_split_acc(D, B1, m);
  const int vb = p.vbits;
  const int hpp = 2 * NW * vb;                 // 16-bit code halves per part

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    mbar_init(&s_aready, TG_EPI / 32);           // one arrival per epilogue warp
    mbar_init(&s_ydone, 1);
    mbar_init(&s_zdone, 1);
    mbar_init(&s_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  if (tid < TC_PARTS * 16) {
    const int pp = tid >> 4, x = tid & 15;
    s_hofs[pp][x] = x < hpp ? code_half_off(p, pp * hpp + x) : 0;
  }
  if (warp == TG_EPI / 32) {
    tc::tmem_alloc(smem_u32(&s_tmem), tcols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const int64_t my_tiles = blockIdx.x < total_tiles ? (total_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == TG_EPI / 32) {
    // ------------------------------------------------ the tensor warp (one thread)
    if (lane == 0) {
      const uint32_t sAH = smem_u32(AH), sAL = smem_u32(AL), sST = smem_u32(ST);
      // when a tile's pieces all fit in the stages they are loaded once and stay
      const bool resident = nC <= NS;
      const int64_t total_p = resident ? nC : my_tiles * nC;
      pdl_wait();                                // the image is written by the previous kernel
      int64_t loaded = 0, gp = 0;
      bool ok = true;
      auto load = [&](int64_t gpc) {
        const int st = (int)(gpc % NS);
        const TgPiece pc = tg_piece((int)(gpc % nC), D, m, NY);
        const uint32_t bytes = (uint32_t)pc.nr * 256u;
        mmadec::mbar_expect_tx(&s_full[st], bytes);
        if (TQ_CHECKED(img + pc.off, bytes, img, img_bytes, 430))
          mmadec::bulk_load(ST + (size_t)st * TG_PIECE, img + pc.off, bytes, &s_full[st]);
      };
      for (; loaded < NS && loaded < total_p; ++loaded) load(loaded);
      uint32_t aph = 0;
      for (int64_t t = 0; t < my_tiles && ok; ++t) {
        for (int pass = B1 > 0 ? 0 : 1; pass < 2 && ok; ++pass) {
          // operand A (U, or E) written by all epilogue threads (polled without a
          // sleep hint: this handoff is on every tile's critical path)
          if (!mbar_wait(&s_aready, aph) || *reinterpret_cast<volatile int*>(&s_abort)) {
            ok = false;
            break;
          }
          aph ^= 1u;
          tc::fence_after_sync();
          const int c0 = pass == 0 ? 0 : NY, c1 = pass == 0 ? NY : nC;
          for (int c = c0; c < c1; ++c, ++gp) {
            const int st = resident ? c : (int)(gp % NS);
            if ((!resident || gp < nC) && !mbar_wait(&s_full[st], (uint32_t)((gp / NS) & 1))) {
              ok = false;
              break;
            }
            const TgPiece pc = tg_piece(c, D, m, NY);
            const uint32_t idesc = tc::idesc_f16(TCM, pc.nr);
            const uint32_t bh = sST + (uint32_t)st * TG_PIECE, bl = bh + (uint32_t)pc.nr * 128u;
            const uint32_t dt = tmem + (uint32_t)pc.dcol;
            const uint32_t dc = split ? dt + tcols / 2 : dt;     // corrections
#pragma unroll
            for (int ks = 0; ks < TG_KC / 16; ++ks) {
              const uint32_t ao = (uint32_t)pc.kc * 1024u + 256u * ks, bo = 256u * ks;
              const uint64_t dah = tc::smem_desc_sbo(sAH + ao, 16 * D), dal = tc::smem_desc_sbo(sAL + ao, 16 * D);
              const uint64_t dbh = tc::smem_desc_sbo(bh + bo, 1024), dbl = tc::smem_desc_sbo(bl + bo, 1024);
              const uint32_t first = (pc.kc | ks) ? 1u : 0u;
              tc::mma_f16(dt, dah, dbh, idesc, first);
              tc::mma_f16(dc, dah, dbl, idesc, split ? first : 1u);
              tc::mma_f16(dc, dal, dbh, idesc, 1u);
            }
            if (resident) continue;
            tc::mma_commit(smem_u32(&s_empty[st]));
            if (gp >= 1 && loaded < total_p) {
              // refill the previous piece's stage once its products are done
              const int64_t pr = gp - 1;
              if (!mbar_wait(&s_empty[pr % NS], (uint32_t)((pr / NS) & 1))) {
                ++gp;
                ok = false;
                break;
              }
              load(loaded);
              ++loaded;
            }
          }
          if (!ok) break;
          tc::mma_commit(smem_u32(pass == 0 ? &s_ydone : &s_zdone));
        }
      }
      if (!ok) {
        // a wait gave up: let every product and copy in flight finish (bounded)
        s_abort = 1;
        atomicExch(&g_quant_tc_err, 1);
        tc::mma_commit(smem_u32(&s_drain));
        (void)mbar_wait(&s_drain, 0u);
        for (int64_t q = gp; q < loaded; ++q) (void)mbar_wait(&s_full[q % NS], (uint32_t)((q / NS) & 1));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ the epilogue warps
    const int q = warp & 3, part = warp >> 2;
    const int r = 32 * q + lane;                 // this thread's row of every tile
    const int kw0 = part * NW;                   // and its first 32-wide word
    const int g = p.group;
    const uint32_t levels = (1u << vb) - 1u;
    const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
    float bnd[L - 1], cen[L];
#pragma unroll
    for (int k = 0; k < L; ++k) cen[k] = B1 > 0 ? p.cent[k] : 0.f;
#pragma unroll
    for (int k = 0; k + 1 < L; ++k) bnd[k] = B1 > 0 ? p.bnd[k] : 0.f;
    // source rows of a tile: this thread's key and value segments (register copies
    // one tile ahead at D = 128; requests towards L2 at D = 256)
    RawSeg<F32> xr[NW], vr[NW];
    auto row_src = [&](int64_t t, bool values, int64_t& e) -> const void* {
      if (t >= total_tiles) return nullptr;
      int64_t ti;
      const int tbh = tile_bh(t, tiles_per_bh, ti);
      ti += r;
      if (ti >= p.n || (values && !p.do_values)) return nullptr;
      return src_row(p, values, tbh, ti, e);
    };
    auto request = [&](int64_t t) {
      int64_t ek = 0, ev = 0;
      const void* ks = row_src(t, false, ek);
      const void* vs = row_src(t, true, ev);
      if constexpr (NW == 1) {
        raw_load(xr[0], ks, ek + 32 * kw0, ks != nullptr);
        raw_load(vr[0], vs, ev + 32 * kw0, vs != nullptr);
      } else {
        const int es = F32 ? 4 : 2;
        if (ks) prefetch_l2(static_cast<const char*>(ks) + (ek + 32 * kw0) * es);
        if (vs) prefetch_l2(static_cast<const char*>(vs) + (ev + 32 * kw0) * es);
      }
    };
    request(blockIdx.x);
    int64_t it = 0;
    for (int64_t tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      int64_t grow;
      const int bh = tile_bh(tile, tiles_per_bh, grow);
      grow += r;
      const bool valid = grow < p.n;
      const uint32_t ph = (uint32_t)(it & 1);
      {
        // the rows of the tile after next towards L2 (this thread's segments)
        int64_t ek = 0, ev = 0;
        const void* ks = row_src(tile + 2 * (int64_t)gridDim.x, false, ek);
        const void* vs = row_src(tile + 2 * (int64_t)gridDim.x, true, ev);
        const int es = F32 ? 4 : 2;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          if (ks) prefetch_l2(static_cast<const char*>(ks) + (ek + 32 * (kw0 + w)) * es);
          if (vs) prefetch_l2(static_cast<const char*>(vs) + (ev + 32 * (kw0 + w)) * es);
        }
      }
      if constexpr (NW > 1) {
        int64_t ek = 0;
        const void* ks = row_src(tile, false, ek);
#pragma unroll
        for (int w = 0; w < NW; ++w) raw_load(xr[w], ks, ek + 32 * (kw0 + w), ks != nullptr);
      }
      // ---- 1. rho and U = X / rho
      float rhof;
      double rho64;
      {
        double ss = 0.0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          float x[32], s8[8];
          raw_to_float(xr[w], p.dtype, x);
#pragma unroll
          for (int j = 0; j < 8; ++j) s8[j] = 0.f;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 xx = make_float2(x[j], x[j + 1]);
            const float2 sp = mmadec::fma2(xx, xx, make_float2(s8[j & 7], s8[(j + 1) & 7]));
            s8[j & 7] = sp.x;
            s8[(j + 1) & 7] = sp.y;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) ss += (double)s8[j];
        }
        ssp[part * TCM + r] = ss;
        tc::bar_sync(1, TG_EPI);
        ss = (ssp[r] + ssp[TCM + r]) + (ssp[2 * TCM + r] + ssp[3 * TCM + r]);
        const double rs = ss > 0.0 ? rsqrt(ss) : 0.0;
        rho64 = ss * rs;
        rhof = (float)rho64;
        const float inv = (float)rs;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          float x[32];
          raw_to_float(xr[w], p.dtype, x);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const float2 u = mmadec::mul2(make_float2(x[8 * c8 + k], x[8 * c8 + k + 1]), make_float2(inv, inv));
              v[k] = u.x;
              v[k + 1] = u.y;
            }
            uint4 hi, lo;
            split8(v, kSplit, hi, lo);
            const int k = 32 * (kw0 + w) + 8 * c8;
            const int off = (((r >> 3) * (D / 8)) + (k >> 3)) * 128 + (r & 7) * 16;
            *reinterpret_cast<uint4*>(AH + off) = hi;
            *reinterpret_cast<uint4*>(AL + off) = lo;
          }
        }
      }
      tc::fence_async_shared();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mmadec::mbar_arrive(&s_aready);
      // ---- 2. values of this thread's 32 NW channels, while the first product runs
      if (p.do_values) {
        if constexpr (NW > 1) {
          int64_t ev = 0;
          const void* vs = row_src(tile, true, ev);
#pragma unroll
          for (int w = 0; w < NW; ++w) raw_load(vr[w], vs, ev + 32 * (kw0 + w), vs != nullptr);
        }
        constexpr int NCH = 2 * NW;                // 16-channel chunks of this thread
        float mn[NCH], mx[NCH];
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          float v[32];
          raw_to_float(vr[w], p.dtype, v);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float a = v[16 * c], b = v[16 * c];
#pragma unroll
            for (int k = 1; k < 16; ++k) {
              a = fminf(a, v[16 * c + k]);
              b = fmaxf(b, v[16 * c + k]);
            }
            mn[2 * w + c] = a;
            mx[2 * w + c] = b;
          }
        }
        const int gc = g / 16;                     // chunks per group
        if (gc <= NCH) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const int c0 = c - c % gc;
            float a = mn[c0], b = mx[c0];
            for (int j = 1; j < gc; ++j) {
              a = fminf(a, mn[c0 + j]);
              b = fmaxf(b, mx[c0 + j]);
            }
            // in place: rewriting a group's first chunk with the group's extremes
            // leaves the later chunks of the group with the same result
            mn[c] = a;
            mx[c] = b;
          }
        } else {
          float a = mn[0], b = mx[0];
#pragma unroll
          for (int c = 1; c < NCH; ++c) {
            a = fminf(a, mn[c]);
            b = fmaxf(b, mx[c]);
          }
          vmm[part * TCM + r] = make_float2(a, b);
          tc::bar_sync(1, TG_EPI);
          const int np = gc / NCH, p0 = part - part % np;
          a = FLT_MAX;
          b = -FLT_MAX;
          for (int j = 0; j < np; ++j) {
            const float2 m2 = vmm[(p0 + j) * TCM + r];
            a = fminf(a, m2.x);
            b = fmaxf(b, m2.y);
          }
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            mn[c] = a;
            mx[c] = b;
          }
        }
        if (valid) {
          float sc[NCH], iv[NCH];
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            sc[c] = __fdiv_rn(__fsub_rn(mx[c], mn[c]), (float)levels);
            iv[c] = sc[c] != 0.f ? __frcp_rn(sc[c]) : 0.f;
          }
          float* vsp = reinterpret_cast<float*>(dst_field(p, bh, grow, 5));
          float* vmp = reinterpret_cast<float*>(dst_field(p, bh, grow, 6));
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const int ch = 32 * kw0 + 16 * c;
            if (ch % g == 0) {
              vsp[ch / g] = sc[c];
              vmp[ch / g] = mn[c];
            }
          }
          uint8_t* cb = code_base(p, bh, grow);
          uint32_t hw[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) hw[j] = 0u;
          bool any_tie = false;
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            float v[32];
            raw_to_float(vr[w], p.dtype, v);
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const int c = 2 * w + (k >> 4);
              bool tie;
              uint32_t c0, c1;
              value_code_pair(v[k], v[k + 1], mn[c], iv[c], levels, c0, c1, tie);
              any_tie |= tie && sc[c] != 0.f;
              const int ch = 32 * w + k;             // channel within this thread's range
              if (vb == 2) hw[ch >> 3] += (c0 << (2 * (ch & 7))) + (c1 << (2 * ((ch + 1) & 7)));
              else hw[ch >> 2] += (c0 << (4 * (ch & 3))) + (c1 << (4 * ((ch + 1) & 3)));
            }
          }
          if (any_tie) {
#pragma unroll
            for (int j = 0; j < 16; ++j) hw[j] = 0u;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
              float v[32];
              raw_to_float(vr[w], p.dtype, v);
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                const int c = 2 * w + (k >> 4), ch = 32 * w + k;
                const uint32_t cd = value_code_fast(v[k], mn[c], sc[c], iv[c], levels);
                if (vb == 2) hw[ch >> 3] += cd << (2 * (ch & 7));
                else hw[ch >> 2] += cd << (4 * (ch & 3));
              }
            }
          }
#pragma unroll
          for (int x = 0; x < 16; ++x)
            if (x < hpp && TQ_CHECKED(cb + s_hofs[part][x], 2, p.cache_mode ? p.base : p.arr.codes,
                                      p.cache_mode ? p.g.total_bytes
                                                   : (p.t_first + p.n) * (p.d * p.vbits / 8), 433))
              *reinterpret_cast<uint16_t*>(cb + s_hofs[part][x]) = (uint16_t)hw[x];
        }
      }
      // the next tile's rows: this tile's register copies are consumed
      request(tile + gridDim.x);
      bool ok = true;
      // ---- 3. codes, E, ||r||
      if constexpr (B1 > 0) {
        ok = !*reinterpret_cast<volatile int*>(&s_abort) && mbar_wait_sleep(&s_ydone, ph);
        if (!ok) {
          s_abort = 1;
          atomicExch(&g_quant_tc_err, 1);
        }
        tc::fence_after_sync();
        uint32_t pw[B1][NW];
        double se = 0.0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          uint32_t acc[32];
          tc::tmem_ld32(trow + (uint32_t)(32 * (kw0 + w)), acc);
          if (split) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {   // the corrections 16 columns at a time
              uint32_t cor[16];
              tc::tmem_ld16(trow + tcols / 2 + (uint32_t)(32 * (kw0 + w)) + 16 * hh, cor);
              tc::tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c)
                acc[16 * hh + c] = __float_as_uint(__uint_as_float(acc[16 * hh + c]) + __uint_as_float(cor[c]));
            }
          }
          tc::tmem_wait_ld();
#pragma unroll
          for (int pl = 0; pl < B1; ++pl) pw[pl][w] = 0u;
          float e[32], s8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) s8[j] = 0.f;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 y2 = mmadec::mul2(make_float2(__uint_as_float(acc[c]), __uint_as_float(acc[c + 1])),
                                           make_float2(1.f / (kSplit * kSplit), 1.f / (kSplit * kSplit)));
            const float yy[2] = {y2.x, y2.y};
            float cv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              int idx;
              code_search<B1>(yy[u], bnd, cen, idx, cv[u]);
#pragma unroll
              for (int pl = 0; pl < B1; ++pl) pw[pl][w] |= (uint32_t)((idx >> pl) & 1) << (c + u);
            }
            const float2 e2 = mmadec::sub2(y2, make_float2(cv[0], cv[1]));
            e[c] = e2.x;
            e[c + 1] = e2.y;
            const float2 sp = mmadec::fma2(e2, e2, make_float2(s8[c & 7], s8[(c + 1) & 7]));
            s8[c & 7] = sp.x;
            s8[(c + 1) & 7] = sp.y;
          }
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = e[8 * c8 + k];
            uint4 hi, lo;
            split8(v, kSplit, hi, lo);
            const int k = 32 * (kw0 + w) + 8 * c8;
            const int off = (((r >> 3) * (D / 8)) + (k >> 3)) * 128 + (r & 7) * 16;
            *reinterpret_cast<uint4*>(AH + off) = hi;
            *reinterpret_cast<uint4*>(AL + off) = lo;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) se += (double)s8[j];
        }
        tc::fence_async_shared();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mmadec::mbar_arrive(&s_aready);
        sep[part * TCM + r] = se;
        tc::bar_sync(3, TG_EPI);
        if (valid && ok) {
          uint8_t* ip = dst_field(p, bh, grow, 0);
#pragma unroll
          for (int pl = 0; pl < B1; ++pl)
#pragma unroll
            for (int w = 0; w < NW; ++w)
              *reinterpret_cast<uint32_t*>(ip + pl * (D / 8) + 4 * (kw0 + w)) = pw[pl][w];
          if (part == 0) {
            const double sev = (sep[r] + sep[TCM + r]) + (sep[2 * TCM + r] + sep[3 * TCM + r]);
            *reinterpret_cast<float*>(dst_field(p, bh, grow, 3)) = (float)(rho64 * sqrt(sev));
          }
        }
      }
      // ---- 4. sign bits of z (rho Z for b1 > 0, S x = rho Z for b1 = 0)
      ok = ok && !*reinterpret_cast<volatile int*>(&s_abort) && mbar_wait_sleep(&s_zdone, ph);
      if (!ok) {
        s_abort = 1;
        atomicExch(&g_quant_tc_err, 1);
      }
      tc::fence_after_sync();
      {
        uint8_t* sp = valid && ok ? dst_field(p, bh, grow, 1) : nullptr;
        for (int w = part; w < m / 32; w += TC_PARTS) {
          uint32_t acc[32];
          tc::tmem_ld32(trow + (uint32_t)(32 * w), acc);
          if (split) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {   // the corrections 16 columns at a time
              uint32_t cor[16];
              tc::tmem_ld16(trow + tcols / 2 + (uint32_t)(32 * w) + 16 * hh, cor);
              tc::tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c)
                acc[16 * hh + c] = __float_as_uint(__uint_as_float(acc[16 * hh + c]) + __uint_as_float(cor[c]));
            }
          }
          tc::tmem_wait_ld();
          // bit = [z >= 0]: [Z >= 0] for rho > 0 (a set-on-compare mask per column);
          // a zero rho makes z = 0, every bit 1
          uint32_t pos = 0u;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            uint32_t mk;
            asm("set.ge.u32.f32 %0, %1, 0f00000000;" : "=r"(mk) : "f"(__uint_as_float(acc[c])));
            pos |= mk & (1u << c);
          }
          if (sp) *reinterpret_cast<uint32_t*>(sp + 4 * w) = rhof > 0.f ? pos : 0xFFFFFFFFu;
        }
        if (sp && part == 0) *reinterpret_cast<float*>(dst_field(p, bh, grow, 2)) = rhof;
      }
      tc::fence_before_sync();
      tc::bar_sync(4, TG_EPI);
      if (*reinterpret_cast<volatile int*>(&s_abort)) break;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == TG_EPI / 32) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, tcols);
  }
}

}  // namespace

// A private stream-ordered memory pool per device for the operand images: freed
// blocks stay in the pool (no release threshold), so the per-call allocation is a
// stream-ordered reuse, never a new mapping.
static cudaError_t image_pool(cudaMemPool_t* out) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = UINT64_MAX;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    pools[dev] = pool;
  }
  *out = pools[dev];
  return cudaSuccess;
}

static cudaError_t run_quantize(QParams& p, int bh_count, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  // the tile kernels index a call's tiles in 32 bits
  const bool tiles32 = (p.n + TCM - 1) / TCM * bh_count < (int64_t)1 << 31;
  if (tiles32 && p.n > 8 && p.do_keys && p.d == QD && p.m == QM && p.b1 > 0 && p.b1 <= 3) {
    // fifth-generation tensor cores: one persistent CTA per SM over 128-token tiles
    const int64_t tiles_per_bh = (p.n + TCM - 1) / TCM;
    const int64_t total = tiles_per_bh * bh_count;
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = tc_smem_bytes();
    const bool f32 = p.dtype == TQ_F32;
    auto kern = p.b1 == 1 ? (f32 ? k_quantize_tc<1, true> : k_quantize_tc<1, false>)
              : p.b1 == 2 ? (f32 ? k_quantize_tc<2, true> : k_quantize_tc<2, false>)
                          : (f32 ? k_quantize_tc<3, true> : k_quantize_tc<3, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = total < sms ? total : sms;
    // a cache append whose chunk replaces the whole ring writes the ring in this
    // kernel, which is then launched programmatically: consecutive appends overlap
    p.fuse_ring = p.cache_mode && p.g.W > 0 && p.n_new >= p.g.W;
    if (p.fuse_ring) return launch_pdl(kern, dim3((unsigned)grid), dim3(TC_THREADS), smem, s, p, tiles_per_bh, total);
    kern<<<(unsigned)grid, TC_THREADS, smem, s>>>(p, tiles_per_bh, total);
    return cudaGetLastError();
  }
  if (tiles32 && p.n > 8 && p.do_keys && (p.d == 128 || p.d == 256) && p.m % 32 == 0 && p.m <= 512 &&
      p.b1 >= 0 && p.b1 <= 3) {
    // the same on streamed operand pieces: Pi and T written once into a scratch image
    const int64_t tiles_per_bh = (p.n + TCM - 1) / TCM;
    const int64_t total = tiles_per_bh * bh_count;
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ib = (int64_t)tg_image_bytes(p.d, p.b1, p.m);
    void* img = nullptr;
    cudaMemPool_t pool;
    cudaError_t e = image_pool(&pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&img, (size_t)ib, pool, s);
    if (e != cudaSuccess) return e;
    const int64_t chunks = (int64_t)((p.b1 > 0 ? p.d : 0) + p.m) * (p.d / 8);
    k_operand_image<<<(unsigned)((chunks + 255) / 256), 256, 0, s>>>(p.Pi, p.T, p.d, p.b1, p.m,
                                                                     static_cast<uint8_t*>(img), ib);
    e = cudaGetLastError();
    if (e == cudaSuccess) {
      const bool f32 = p.dtype == TQ_F32, wide = p.d == 256;
      using KFn = void (*)(QParams, const uint8_t*, int64_t, int64_t, int64_t);
      static const KFn table[2][4][2] = {
          {{k_quantize_tcg<128, 0, false>, k_quantize_tcg<128, 0, true>},
           {k_quantize_tcg<128, 1, false>, k_quantize_tcg<128, 1, true>},
           {k_quantize_tcg<128, 2, false>, k_quantize_tcg<128, 2, true>},
           {k_quantize_tcg<128, 3, false>, k_quantize_tcg<128, 3, true>}},
          {{k_quantize_tcg<256, 0, false>, k_quantize_tcg<256, 0, true>},
           {k_quantize_tcg<256, 1, false>, k_quantize_tcg<256, 1, true>},
           {k_quantize_tcg<256, 2, false>, k_quantize_tcg<256, 2, true>},
           {k_quantize_tcg<256, 3, false>, k_quantize_tcg<256, 3, true>}}};
      const KFn kern = table[wide][p.b1][f32];
      const size_t smem = tg_smem_bytes();
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) {
        const int64_t grid = total < sms ? total : sms;
        e = launch_pdl(kern, dim3((unsigned)grid), dim3(TG_THREADS), smem, s, p,
                       static_cast<const uint8_t*>(img), ib, tiles_per_bh, total);
      }
    }
    const cudaError_t ef = cudaFreeAsync(img, s);
    return e != cudaSuccess ? e : ef;
  }
  if (p.n <= 8) {
    // a few tokens per (b, kv head): one CTA per token
    const size_t smem = sizeof(float) * (2 * p.d + (p.m > p.d ? p.m : p.d) + 32);
    dim3 grid((unsigned)p.n, (unsigned)bh_count, 2);
    k_quantize_small<<<grid, SMALL_THREADS, smem, s>>>(p);
    return cudaGetLastError();
  }
  // 64-token tiles where two CTAs fit an SM, else 32
  const int kb1 = p.do_keys ? p.b1 : 0;
  const int nt = smem_bytes(p.d, 64, kb1) <= (110u << 10) ? 64 : 32;
  const size_t smem = smem_bytes(p.d, nt, kb1);
  auto kern = nt == 32 ? k_quantize<32> : k_quantize<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.n + nt - 1) / nt), (unsigned)bh_count);
  kern<<<grid, THREADS, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t quantize_error_flag(int* flag, cudaStream_t s) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(flag, g_quant_tc_err, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_quant_tc_err, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e;
}

cudaError_t launch_quantize_arrays(const QuantSrc& src, int dtype, int d, int b1, int m,
                                   int vbits, int group, bool do_keys, bool do_values,
                                   const float* Pi, const float* T, const float* cent,
                                   const float* bnd, const QuantDst& dst, cudaStream_t s) {
  QParams p{};
  p.K = src.K;
  p.V = src.V;
  p.dtype = dtype;
  p.n = src.n;
  p.t_first = 0;
  p.cache_mode = false;
  p.d = d;
  p.b1 = b1;
  p.m = m;
  p.vbits = vbits;
  p.group = group;
  p.do_keys = do_keys;
  p.do_values = do_values;
  p.Pi = Pi;
  p.T = T;
  p.cent = cent;
  p.bnd = bnd;
  p.arr = dst;
  return run_quantize(p, 1, s);
}

cudaError_t launch_quantize_cache(const QuantSrc& src, const Geom& g, uint8_t* base,
                                  const float* Pi, const float* T, const float* cent,
                                  const float* bnd, cudaStream_t s, bool* ring_written) {
  QParams p{};
  p.K = src.K;
  p.V = src.V;
  p.dtype = g.dtype;
  p.n = src.n;
  p.t_first = src.t_first;
  p.n_old = src.n_old;
  p.n_new = src.n_new;
  p.cache_mode = true;
  p.ringK = base + g.ring_k_off;
  p.ringV = base + g.ring_v_off;
  p.d = g.d;
  p.b1 = g.b1;
  p.m = g.m;
  p.vbits = g.vbits;
  p.group = g.group;
  p.do_keys = true;
  p.do_values = true;
  p.Pi = Pi;
  p.T = T;
  p.cent = cent;
  p.bnd = bnd;
  p.base = base;
  p.g = g;
  p.hadamard = g.hadamard;
  const cudaError_t e = run_quantize(p, g.B * g.Hkv, s);
  if (ring_written) *ring_written = e == cudaSuccess && p.fuse_ring;
  return e;
}

cudaError_t launch_ring_write(const Geom& g, uint8_t* base, const void* K, const void* V,
                              int64_t n_old, int64_t n_new, cudaStream_t s) {
  if (g.W == 0 || n_new == 0) return cudaSuccess;
  return launch_pdl(k_ring_write, dim3(g.B * g.Hkv), dim3(256), 0, s, g, base, K, V, n_old, n_new);
}

cudaError_t launch_decode_step_pre(const QuantSrc& src, int64_t n_ring_only, const Geom& g,
                                   uint8_t* base, const float* Pi, const float* T,
                                   const float* cent, const float* bnd, const void* Q, int Hq,
                                   const float* S, float softmax_scale, const DecodeWs& ws,
                                   cudaStream_t s) {
  QParams p{};
  p.K = src.K;
  p.V = src.V;
  p.dtype = g.dtype;
  p.n = src.n;
  p.t_first = src.t_first;
  p.n_old = src.n_old;
  p.n_new = src.n_new;
  p.cache_mode = true;
  p.ringK = base + g.ring_k_off;
  p.ringV = base + g.ring_v_off;
  p.d = g.d;
  p.b1 = g.b1;
  p.m = g.m;
  p.vbits = g.vbits;
  p.group = g.group;
  p.do_keys = true;
  p.do_values = true;
  p.Pi = Pi;
  p.T = T;
  p.cent = cent;
  p.bnd = bnd;
  p.base = base;
  p.g = g;
  p.hadamard = g.hadamard;
  const int units = g.B * g.Hkv;
  const int nq = (int)(src.n * units * 2), nr = (int)(n_ring_only * units);
  StepPrep sp{g, Q, Hq, Pi, S, cent, softmax_scale * mmadec::kLog2e, ws};
  const size_t qsm = sizeof(float) * (2 * g.d + (g.m > g.d ? g.m : g.d) + 32);
  const size_t psm = mmadec::prep_smem_bytes(g.d, g.m);
  const size_t smem = qsm > psm ? qsm : psm;
  auto kern = g.d == 256 ? k_step_pre<2> : k_step_pre<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<nq + nr + 2 * units, SMALL_THREADS, smem, s>>>(p, nq, nr, sp);   // prep: 2 halves a unit
  return cudaGetLastError();
}

TQ_BOUNDS_READER(bounds_flag_quant)

}  // namespace tq
