// Key/value quantisation and append ([TQ] 二 three-stage pipeline, 五
// ProdQuantized, 六 store + ring, 七 value group quantisation).
//
// One CTA quantises a tile of 64 tokens of one (b, kv head):
//   keys   rho = ||x|| (float64 sum of exact fp32 squares)
//          Y = X Pi^T (fp32 FMA), y = Y / rho, idx_j = #{k : beta_k < y_j},
//          e = y - c[idx], ||r|| = rho ||e||, z = rho (T e) with T = S Pi^T,
//          sign bit = [z >= 0]; bit-planes and signs packed with warp ballots
//          (lane i -> bit i, so words are LSB-first / little-endian).
//          Pure QJL (b1 = 0): z = S x.
//   values per (token, group): mn, mx, s = (mx - mn)/(2^vb - 1),
//          code = clamp(rint((v - mn)/s)) in IEEE fp32 (__fsub_rn/__fdiv_rn/rintf).
// The contractions run as a register-tiled fp32 SGEMM (64 tokens x 128 columns
// per pass, 4x8 outputs per thread).
#include <cfloat>

#include "common.cuh"
#include "prep_mma.cuh"

namespace tq {
namespace {

constexpr int NT = 64;        // tokens per tile
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
  const void* ringK;
  const void* ringV;
  // shapes
  int d, b1, m, vbits, group;
  bool do_keys, do_values;
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
  float* X;      // [NT][d+4]
  float* Y;      // [NT][d+4]
  float* B;      // [KC][SBS]
  float* Z;      // [NT][SBS]
  double* rho64; // [NT]
  float* rho;    // [NT]
  float* inv;    // [NT]
  float* cb;     // [16] centroids, [16] boundaries
  float* vs;     // [NT * 16] value scales
  float* vm;     // [NT * 16] value minima
};

__host__ __device__ inline size_t smem_bytes(int d) {
  const int sx = d + 4;
  return sizeof(float) * (2 * NT * sx + KC * SBS + NT * SBS) + sizeof(double) * NT +
         sizeof(float) * (2 * NT + 32 + 2 * NT * 16);
}

__device__ Smem carve(unsigned char* raw, int d) {
  Smem s;
  const int sx = d + 4;
  double* dp = reinterpret_cast<double*>(raw);
  s.rho64 = dp;
  float* f = reinterpret_cast<float*>(dp + NT);
  s.X = f;
  f += NT * sx;
  s.Y = f;
  f += NT * sx;
  s.B = f;
  f += KC * SBS;
  s.Z = f;
  f += NT * SBS;
  s.rho = f;
  f += NT;
  s.inv = f;
  f += NT;
  s.cb = f;
  f += 32;
  s.vs = f;
  f += NT * 16;
  s.vm = f;
  return s;
}

// Element pointer base + index of row i (token t_first + i) of (b, h) in the source.
__device__ __forceinline__ const void* src_row(const QParams& p, bool values, int bh, int64_t i,
                                               int64_t& elem) {
  const int d = p.d;
  const void* chunk = values ? p.V : p.K;
  if (!p.cache_mode) {
    elem = i * d;
    return chunk;
  }
  const int64_t t = p.t_first + i;
  if (t < p.n_old) {
    elem = ((int64_t)bh * p.g.W + t % p.g.W) * d;
    return values ? p.ringV : p.ringK;
  }
  elem = ((int64_t)bh * p.n_new + (t - p.n_old)) * d;
  return chunk;
}

// 16-bit half x (codes of channels (16/vbits) x ...) of the value codes of row i:
// token-major in the standalone arrays, token-pair records in the cache.
__device__ __forceinline__ uint16_t* code_half_ptr(const QParams& p, int bh, int64_t i, int x) {
  if (p.cache_mode) {
    const Geom& g = p.g;
    const int64_t t = p.t_first + i;
    uint8_t* blk = p.base + (int64_t)bh * g.region_bytes + (t / kBlockTokens) * g.block_bytes;
    return reinterpret_cast<uint16_t*>(blk + g.o_vcode + vcode_half_off(g, (int)(t % kBlockTokens), x));
  }
  return reinterpret_cast<uint16_t*>(p.arr.codes + (p.t_first + i) * (p.d * p.vbits / 8)) + x;
}

__device__ __forceinline__ uint8_t* dst_field(const QParams& p, int bh, int64_t i, int which) {
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

// acc[r][c] = sum_k A[4ty+r][k] * Bg[col0 + tx + 16c][k], k < kdim; Bg row-major
// [ncols][kdim], rows past ncols read as zero.
__device__ void gemm_pass(const float* A, int sa, const float* Bg, int kdim, int col0, int ncols,
                          float* sB, float acc[4][8]) {
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
#pragma unroll
  for (int r = 0; r < 4; ++r)
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
      float a[4], b[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = A[(4 * ty + r) * sa + k0 + kk];
#pragma unroll
      for (int c = 0; c < 8; ++c) b[c] = sB[kk * SBS + tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
}

__device__ void quantize_keys_tile(const QParams& p, const Smem& s, int bh, int64_t row0) {
  const int d = p.d, sx = d + 4, b1 = p.b1, m = p.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ty = tid / 16, tx = tid % 16;
  load_tile(p, false, bh, row0, s.X);
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
    for (int col0 = 0; col0 < d; col0 += NC) {
      float acc[4][8];
      gemm_pass(s.X, sx, p.Pi, d, col0, d, s.B, acc);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int col = col0 + tx + 16 * c;
          if (col < d) s.Y[(4 * ty + r) * sx + col] = acc[r][c] * s.inv[4 * ty + r];
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
    float acc[4][8];
    gemm_pass(E, sx, p.T, d, col0, m, s.B, acc);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float z = (b1 > 0) ? acc[r][c] * s.rho[4 * ty + r] : acc[r][c];
        s.Z[(4 * ty + r) * SBS + tx + 16 * c] = z;
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

__device__ void quantize_values_tile(const QParams& p, const Smem& s, int bh, int64_t row0) {
  const int d = p.d, sx = d + 4, g = p.group, ng = d / g, vb = p.vbits;
  const float levels = (float)((1 << vb) - 1);
  const int tid = threadIdx.x;
  load_tile(p, true, bh, row0, s.X);
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

__global__ void __launch_bounds__(THREADS) k_quantize(QParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem s = carve(smem_raw, p.d);
  const int bh = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * NT;
  if (threadIdx.x < 16) {
    const int L = p.b1 > 0 ? (1 << p.b1) : 0;
    s.cb[threadIdx.x] = (threadIdx.x < L) ? p.cent[threadIdx.x] : 0.f;
    s.cb[16 + threadIdx.x] = (threadIdx.x + 1 < L) ? p.bnd[threadIdx.x] : 0.f;
  }
  __syncthreads();
  if (p.do_keys) quantize_keys_tile(p, s, bh, row0);
  __syncthreads();
  if (p.do_values) quantize_values_tile(p, s, bh, row0);
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
    dst[w] = src[w];
  }
}

// One CTA per token and per half (blockIdx.z = 0: key, 1: value), for launches
// with only a few tokens per (b, kv head) (the decode step appends one): the
// same arithmetic as the 64-token tile.  The key CTA runs its matrix-vector
// products two threads per row (each streams half the row as float4, the vector
// is a shared-memory broadcast) and reduces rho while Pi x is being formed.
constexpr int SMALL_THREADS = 256;

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
        if (b1 > 0)
          for (int c = half * (d / 2); c < (half + 1) * (d / 2); c += 32) prefetch_l2(p.Pi + (int64_t)j * d + c);
      for (int a = tid >> 1; a < m; a += SMALL_THREADS / 2)
        for (int c = half * (d / 2); c < (half + 1) * (d / 2); c += 32) prefetch_l2(p.T + (int64_t)a * d + c);
    }
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
    if (ring_new)    // the token is in shared memory: its ring slot takes the new one
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
      for (int j = tid >> 1; j < d; j += SMALL_THREADS / 2) {
        const float a = half_row_dot(p.Pi + (int64_t)j * d, sx, d, half);
        if (half == 0) sy[j] = a * inv;
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
    for (int a = tid >> 1; a < m; a += SMALL_THREADS / 2) {
      const float acc = half_row_dot(p.T + (int64_t)a * d, E, d, half);
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
    if (ring_new)
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
  mmadec::prep_mma_body<NV>(sp.g, sp.Q, sp.Hq, sp.Pi, sp.S, sp.cent, sp.scale_log2, sp.ws, bid,
                            smem_raw);
}

// ---------------------------------------------------------------------------
// Tensor-core tile path (head dim 128, b1 > 0, m = 128): a persistent CTA per SM
// keeps Pi and T = S Pi^T resident in shared memory as fp16 hi/lo pairs
// (v * 2^10 = hi + lo, |lo| <= 2^-11 |hi|), and loops over 64-token tiles:
//   U = X / rho -> fp16 hi/lo;  Y = U Pi^T  and  Z = E T^T (E = Y - c[idx])
// each as three mma.sync m16n8k16 products (hi*hi + hi*lo + lo*hi, fp32
// accumulate), i.e. about 22 significant bits: well inside the 1e-5 band that
// separates a code or a sign from its decision boundary.
// ---------------------------------------------------------------------------
constexpr int QD = 128;             // head dim of this path
constexpr int QM = 128;             // sketch rows of this path
constexpr int HS = QD + 8;          // fp16 row stride (272 B: conflict-free ldmatrix)
constexpr int YS = QD + 4;          // fp32 row stride of the Y / Z / V tile
constexpr float kSplit = 1024.f;

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void split_store(__half* hi, __half* lo, float v) {
  const float x = v * kSplit;
  const __half h = __float2half_rn(x);
  *hi = h;
  *lo = __float2half_rn(x - __half2float(h));
}

constexpr int QG = 4;              // independent warp groups per CTA
constexpr int QNT = 16;            // rows of a group's tile

struct MmaGroupSmem {
  __half *AH, *AL;                 // [QNT][HS]
  float* YZ;                       // [QNT][YS]
  double* rho64;                   // [QNT]
  float* rho;                      // [QNT]
};

struct MmaSmem {
  __half *PH, *PL, *TH, *TL;       // [128][HS] each
  float* cb;                       // [32]
};

__host__ __device__ inline size_t mma_group_bytes() {
  return sizeof(__half) * 2 * QNT * HS + sizeof(float) * QNT * YS + sizeof(double) * QNT +
         sizeof(float) * QNT;
}

__host__ __device__ inline size_t mma_smem_bytes() {
  return sizeof(__half) * 4 * 128 * HS + QG * mma_group_bytes() + sizeof(float) * 32;
}

__device__ MmaSmem mma_carve(unsigned char* raw) {
  MmaSmem s;
  s.PH = reinterpret_cast<__half*>(raw);
  s.PL = s.PH + 128 * HS;
  s.TH = s.PL + 128 * HS;
  s.TL = s.TH + 128 * HS;
  s.cb = reinterpret_cast<float*>(raw + sizeof(__half) * 4 * 128 * HS + QG * mma_group_bytes());
  return s;
}

__device__ MmaGroupSmem mma_group_carve(unsigned char* raw, int grp) {
  MmaGroupSmem m;
  unsigned char* q = raw + sizeof(__half) * 4 * 128 * HS + (size_t)grp * mma_group_bytes();
  m.AH = reinterpret_cast<__half*>(q);
  m.AL = m.AH + QNT * HS;
  m.YZ = reinterpret_cast<float*>(m.AL + QNT * HS);
  m.rho64 = reinterpret_cast<double*>(m.YZ + QNT * YS);
  m.rho = reinterpret_cast<float*>(m.rho64 + QNT);
  return m;
}

constexpr int QTHREADS = 512;       // 16 warps per CTA on the tensor-core tile path

// C[QNT x 128] = A[QNT x 128] * B^T for one warp group, A and B as fp16 hi/lo
// pairs (rows of 128, stride HS); warp gw (of the group's GW) owns the QNT rows
// and columns (128 / GW) gw .. +128 / GW.  The result (scaled back by 2^-20) goes
// to C (fp32, stride YS).
template <int MTI, int NTI>     // 16-row m-tiles, 16-column B loads per warp
__device__ __forceinline__ void mma_gemm_group(const __half* AH, const __half* AL, const __half* BH,
                                               const __half* BL, float* C, int gw) {
  const int lane = threadIdx.x & 31;
  const int c0 = 16 * NTI * gw;
  float acc[MTI][2 * NTI][4];
#pragma unroll
  for (int i = 0; i < MTI; ++i)
#pragma unroll
    for (int j = 0; j < 2 * NTI; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;
  const int ar = lane & 15, ac = 8 * (lane >> 4);                    // A: rows, k offset
  const int bn = (lane & 7) + 8 * (lane >> 4), bk = 8 * ((lane >> 3) & 1);   // B: n, k offset
#pragma unroll 2
  for (int ks = 0; ks < QD / 16; ++ks) {
    uint32_t ah[MTI][4], al[MTI][4];
#pragma unroll
    for (int i = 0; i < MTI; ++i) {
      ldsm_x4(ah[i], AH + (16 * i + ar) * HS + 16 * ks + ac);
      ldsm_x4(al[i], AL + (16 * i + ar) * HS + 16 * ks + ac);
    }
#pragma unroll
    for (int jb = 0; jb < NTI; ++jb) {
      uint32_t bh[4], bl[4];
      ldsm_x4(bh, BH + (c0 + 16 * jb + bn) * HS + 16 * ks + bk);
      ldsm_x4(bl, BL + (c0 + 16 * jb + bn) * HS + 16 * ks + bk);
#pragma unroll
      for (int i = 0; i < MTI; ++i) {
        mma16816(acc[i][2 * jb], ah[i], bh[0], bh[1]);
        mma16816(acc[i][2 * jb], ah[i], bl[0], bl[1]);
        mma16816(acc[i][2 * jb], al[i], bh[0], bh[1]);
        mma16816(acc[i][2 * jb + 1], ah[i], bh[2], bh[3]);
        mma16816(acc[i][2 * jb + 1], ah[i], bl[2], bl[3]);
        mma16816(acc[i][2 * jb + 1], al[i], bh[2], bh[3]);
      }
    }
  }
  const int gid = lane >> 2, tig = lane & 3;
  const float sc = 1.f / (kSplit * kSplit);
#pragma unroll
  for (int i = 0; i < MTI; ++i)
#pragma unroll
    for (int j = 0; j < 2 * NTI; ++j) {
      const int row = 16 * i + gid, col = c0 + 8 * j + 2 * tig;
      C[row * YS + col] = acc[i][j][0] * sc;
      C[row * YS + col + 1] = acc[i][j][1] * sc;
      C[(row + 8) * YS + col] = acc[i][j][2] * sc;
      C[(row + 8) * YS + col + 1] = acc[i][j][3] * sc;
    }
}

// Values of a warp's rows straight from the source: lane l holds channels
// 4l..4l+3; the group min / max come from xor-shuffles over the g/4 lanes of the
// group; codes leave as one byte (2-bit) or two bytes (4-bit) per lane.
__device__ __forceinline__ void quantize_values_rows(const QParams& p, int bh, int64_t row0, int nrows,
                                                     int warp, int lane, int nwarps) {
  const int d = p.d, g = p.group, vb = p.vbits, lanes_g = g / 4;
  const float levels = (float)((1 << vb) - 1);
  for (int r = warp; r < nrows; r += nwarps) {
    if (row0 + r >= p.n) break;
    int64_t e0;
    const void* src = src_row(p, true, bh, row0 + r, e0);
    float x[4];
    load4(src, e0 + 4 * lane, p.dtype, x);
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    for (int o = 1; o < lanes_g; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
    const float inv = sc != 0.f ? __frcp_rn(sc) : 0.f;
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) bits |= value_code(x[k], mn, sc, inv, levels) << (k * vb);
    if (vb == 2) {
      // a 16-bit half holds the 8 codes of lanes 2x and 2x + 1
      const uint32_t hi = __shfl_down_sync(0xffffffffu, bits, 1);
      if ((lane & 1) == 0) *code_half_ptr(p, bh, row0 + r, lane >> 1) = (uint16_t)(bits | (hi << 8));
    } else {
      *code_half_ptr(p, bh, row0 + r, lane) = (uint16_t)bits;
    }
    if ((lane % lanes_g) == 0) {
      const int gi = (4 * lane) / g;
      reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 5))[gi] = sc;
      reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 6))[gi] = mn;
    }
    (void)d;
  }
}

template <int B1>
__global__ void __launch_bounds__(QTHREADS, 1) k_quantize_mma(QParams p, int64_t tiles_per_bh,
                                                             int64_t total_tiles) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  MmaSmem s = mma_carve(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int L = 1 << B1;
  constexpr int GW = QTHREADS / 32 / QG;         // warps per group
  constexpr int RPW = QNT / GW;                  // rows per warp of a group tile
  // resident operands: Pi and T as fp16 hi/lo, rows of 128 (four elements a thread)
  for (int i = 4 * tid; i < QD * QD; i += 4 * QTHREADS) {
    const int r = i / QD, c = i % QD;
    const float4 a = *reinterpret_cast<const float4*>(p.Pi + i);
    const float4 b = *reinterpret_cast<const float4*>(p.T + i);
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      split_store(s.PH + r * HS + c + k, s.PL + r * HS + c + k, av[k]);
      split_store(s.TH + r * HS + c + k, s.TL + r * HS + c + k, bv[k]);
    }
  }
  if (tid < 16) {
    s.cb[tid] = (tid < L) ? p.cent[tid] : 0.f;
    s.cb[16 + tid] = (tid + 1 < L) ? p.bnd[tid] : 0.f;
  }
  __syncthreads();
  float bnd[L - 1];
#pragma unroll
  for (int k = 0; k + 1 < L; ++k) bnd[k] = s.cb[16 + k];

  // From here the QG warp groups run independently on interleaved QNT-row tiles,
  // each with its own operand / result buffers and its own named barrier, so one
  // group's tensor-core products overlap the other's per-row work.
  const int grp = warp / GW, gw = warp % GW, gtid = tid % (GW * 32);
  const MmaGroupSmem m = mma_group_carve(smem_raw, grp);
  auto group_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(GW * 32) : "memory"); };
  // Bring the key and value rows of a tile towards L2 (one hint per 128-byte line).
  const int es = p.dtype == TQ_F32 ? 4 : 2, lpr = QD * es / 128;
  auto prefetch_tile = [&](int64_t t) {
    if (t >= total_tiles) return;
    const int pbh = (int)(t / tiles_per_bh);
    const int64_t prow0 = (t % tiles_per_bh) * QNT;
    for (int i = gtid; i < QNT * 2 * lpr; i += GW * 32) {
      const int r = i / (2 * lpr), which = (i / lpr) & 1, ln = i % lpr;
      if (prow0 + r >= p.n || (which && !p.do_values)) continue;
      int64_t e0;
      const void* src = src_row(p, which != 0, pbh, prow0 + r, e0);
      prefetch_l2(reinterpret_cast<const char*>(src) + e0 * es + 128 * ln);
    }
  };
  const int64_t t_step = (int64_t)QG * gridDim.x;
  prefetch_tile((int64_t)QG * blockIdx.x + grp);
  for (int64_t tile = (int64_t)QG * blockIdx.x + grp; tile < total_tiles; tile += t_step) {
    const int bh = (int)(tile / tiles_per_bh);
    const int64_t row0 = (tile % tiles_per_bh) * QNT;
    prefetch_tile(tile + t_step);
    // ---- keys: rho (float64), U = X / rho as fp16 hi/lo; a warp's rows are all
    // loaded (4 consecutive elements a lane) before their reductions
    {
      float x[RPW][4];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const int r = gw + i * GW;
        if (row0 + r < p.n) {
          int64_t e0;
          const void* src = src_row(p, false, bh, row0 + r, e0);
          load4(src, e0 + 4 * lane, p.dtype, x[i]);
        } else {
          x[i][0] = x[i][1] = x[i][2] = x[i][3] = 0.f;
        }
      }
      double ss[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        ss[i] = 0.0;
#pragma unroll
        for (int k = 0; k < 4; ++k) ss[i] += (double)x[i][k] * (double)x[i][k];
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) ss[i] = warp_sum_d(ss[i]);
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const int r = gw + i * GW;
        // rho = ss * rsqrt(ss) and 1/rho = rsqrt(ss): one float64 reciprocal square
        // root instead of a square root and a division
        const double rs = ss[i] > 0.0 ? rsqrt(ss[i]) : 0.0;
        const double rho = ss[i] * rs;
        const float inv = (float)rs;
        if (lane == 0) {
          m.rho64[r] = rho;
          m.rho[r] = (float)rho;
        }
        // this lane's 4 consecutive elements: hi / lo as two f16x2 pairs each
        float a[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) a[k] = x[i][k] * inv * kSplit;
        const __half2 h01 = __floats2half2_rn(a[0], a[1]), h23 = __floats2half2_rn(a[2], a[3]);
        const float2 b01 = __half22float2(h01), b23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(a[0] - b01.x, a[1] - b01.y);
        const __half2 l23 = __floats2half2_rn(a[2] - b23.x, a[3] - b23.y);
        uint2 hv, lv;
        hv.x = *reinterpret_cast<const uint32_t*>(&h01);
        hv.y = *reinterpret_cast<const uint32_t*>(&h23);
        lv.x = *reinterpret_cast<const uint32_t*>(&l01);
        lv.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(m.AH + r * HS + 4 * lane) = hv;
        *reinterpret_cast<uint2*>(m.AL + r * HS + 4 * lane) = lv;
      }
    }
    group_sync();
    mma_gemm_group<QNT / 16, 128 / 16 / GW>(m.AH, m.AL, s.PH, s.PL, m.YZ, gw);   // Y = U Pi^T
    group_sync();
    // ---- codes, residual E (fp16 hi/lo into A), ||r||: a warp's rows, lane =
    // coordinate within each 32-coordinate chunk; the plane words of a row are
    // collected by ballot and stored as one 16-byte write per plane
    {
      double se[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const int r = gw + i * GW;
        se[i] = 0.0;
        uint32_t pw[B1][QD / 32];
#pragma unroll
        for (int c = 0; c < QD / 32; ++c) {
          const float y = m.YZ[r * YS + 32 * c + lane];
          int idx = 0;
#pragma unroll
          for (int k = 0; k + 1 < L; ++k) idx += (bnd[k] < y) ? 1 : 0;
          const float e = y - s.cb[idx];
          se[i] += (double)e * (double)e;
          split_store(m.AH + r * HS + 32 * c + lane, m.AL + r * HS + 32 * c + lane, e);
#pragma unroll
          for (int pl = 0; pl < B1; ++pl) pw[pl][c] = __ballot_sync(0xffffffffu, (idx >> pl) & 1);
        }
        if (lane < B1 && row0 + r < p.n) {
          uint4 v = make_uint4(pw[0][0], pw[0][1], pw[0][2], pw[0][3]);
#pragma unroll
          for (int pl = 1; pl < B1; ++pl)
            if (lane == pl) v = make_uint4(pw[pl][0], pw[pl][1], pw[pl][2], pw[pl][3]);
          *reinterpret_cast<uint4*>(dst_field(p, bh, row0 + r, 0) + lane * (QD / 8)) = v;
        }
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) se[i] = warp_sum_d(se[i]);
      if (lane < RPW) {
        // lane i writes row gw + GW i (a constant-index select, no dynamic register index)
        double sv = se[0];
#pragma unroll
        for (int i = 1; i < RPW; ++i)
          if (lane == i) sv = se[i];
        const int r = gw + lane * GW;
        if (row0 + r < p.n) {
          *reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 3)) = (float)(m.rho64[r] * sqrt(sv));
          *reinterpret_cast<float*>(dst_field(p, bh, row0 + r, 2)) = m.rho[r];
        }
      }
    }
    group_sync();
    mma_gemm_group<QNT / 16, 128 / 16 / GW>(m.AH, m.AL, s.TH, s.TL, m.YZ, gw);   // Z = E T^T
    group_sync();
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const int r = gw + i * GW;
      const float rho = m.rho[r];
      uint32_t sw[QM / 32];
#pragma unroll
      for (int c = 0; c < QM / 32; ++c) sw[c] = __ballot_sync(0xffffffffu, m.YZ[r * YS + 32 * c + lane] * rho >= 0.f);
      if (lane == 0 && row0 + r < p.n)
        *reinterpret_cast<uint4*>(dst_field(p, bh, row0 + r, 1)) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
    }
    // ---- values, straight from the source rows
    if (p.do_values) quantize_values_rows(p, bh, row0, QNT, gw, lane, GW);
    group_sync();
  }
}

}  // namespace

static cudaError_t run_quantize(QParams& p, int bh_count, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  if (p.n > 8 && p.do_keys && p.d == QD && p.m == QM && p.b1 > 0) {
    // tensor-core tiles: one persistent CTA per SM, QG warp groups over all
    // QNT-token tiles
    const int64_t tiles_per_bh = (p.n + QNT - 1) / QNT;
    const int64_t total = tiles_per_bh * bh_count;
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = mma_smem_bytes();
    auto kern = p.b1 == 1 ? k_quantize_mma<1> : p.b1 == 2 ? k_quantize_mma<2> : k_quantize_mma<3>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t want = (total + QG - 1) / QG;
    const int64_t grid = want < sms ? want : sms;
    kern<<<(unsigned)grid, QTHREADS, smem, s>>>(p, tiles_per_bh, total);
    return cudaGetLastError();
  }
  if (p.n <= 8) {
    // a few tokens per (b, kv head): one CTA per token
    const size_t smem = sizeof(float) * (2 * p.d + (p.m > p.d ? p.m : p.d) + 32);
    dim3 grid((unsigned)p.n, (unsigned)bh_count, 2);
    k_quantize_small<<<grid, SMALL_THREADS, smem, s>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = smem_bytes(p.d);
  cudaError_t e = cudaFuncSetAttribute(k_quantize, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.n + NT - 1) / NT), (unsigned)bh_count);
  k_quantize<<<grid, THREADS, smem, s>>>(p);
  return cudaGetLastError();
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
                                  const float* bnd, cudaStream_t s) {
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
  return run_quantize(p, g.B * g.Hkv, s);
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
  const int units = g.B * g.Hkv;
  const int nq = (int)(src.n * units * 2), nr = (int)(n_ring_only * units);
  StepPrep sp{g, Q, Hq, Pi, S, cent, softmax_scale * mmadec::kLog2e, ws};
  const size_t qsm = sizeof(float) * (2 * g.d + (g.m > g.d ? g.m : g.d) + 32);
  const size_t psm = mmadec::prep_smem_bytes(g.d, g.m);
  const size_t smem = qsm > psm ? qsm : psm;
  auto kern = g.d == 256 ? k_step_pre<2> : k_step_pre<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<nq + nr + units, SMALL_THREADS, smem, s>>>(p, nq, nr, sp);
  return cudaGetLastError();
}

}  // namespace tq
