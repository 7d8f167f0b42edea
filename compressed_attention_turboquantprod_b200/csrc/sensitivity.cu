// Sensitivity profile of the adaptive per-layer-group sketch dimension ([AQJL]
// sensitivity analyser: each layer's key variance on calibration data decides
// the layer groups and their bit allocation).
//
// Device: the mean and population variance of every entry of a layer's
// calibration keys, one streaming pass at HBM speed.  Entries are taken
// relative to a shift c (the fp32 mean of the first min(n, 32) entries, the
// same in every CTA), so the sums stay of the size of the spread and not of
// the mean: d = x - c, S1 = sum d, S2 = sum d^2, mean = c + S1/n, variance =
// S2/n - (S1/n)^2 (shifted-data formula; the one-pass sum of squares, which
// cancels catastrophically for keys whose mean is large against their spread,
// is never formed).  16-byte loads, d, its sums and its squares in fp64 (all
// exact but the sums), fixed-order block and grid reductions (the result does
// not depend on scheduling).
//
// Host: the groups and sketch dims from the per-layer variances.
//   * contiguous groups whose boundaries minimise the summed squared deviation
//     of the layer variances from their group means (exact dynamic programme;
//     equal optima resolved to the lexicographically smallest boundaries);
//   * sketch dims minimising sum_g n_g s_g / m_g (the QJL term's variance is
//     proportional to |k|^2 / m, [TQ] 四) under sum_g n_g m_g <= L m_avg, each a
//     multiple of 32 in [m_min, m_max]: from m_min, 32 at a time to the group
//     whose step lowers the objective most per sign bit (equal: lower group).
// The sums are sequential IEEE double, so the integer outcome is reproducible.
#include <cmath>
#include <vector>

#include "common.cuh"

namespace tq {
namespace {

constexpr int kMomBlocks = 148 * 4;
constexpr int kMomThreads = 256;
constexpr int kMomUnroll = 4;     // 16-byte loads in flight per thread

// One 16-byte load: d = x - c, its sum and its square in fp64 (x and c are fp32
// values, so d and d^2 are exact in fp64; fp32 squares would round with a bias
// when the entries sit on a coarse grid, as 16-bit inputs do).
__device__ __forceinline__ void moments16(uint4 u, int dtype, double c, double& s1, double& s2) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if (dtype == TQ_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double x = (double)__uint_as_float(w[i]) - c;
      s1 += x;
      s2 = fma(x, x, s2);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float lo, hi;
      if (dtype == TQ_BF16) {
        lo = __uint_as_float(w[i] << 16);
        hi = __uint_as_float(w[i] & 0xFFFF0000u);
      } else {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
        const float2 f = __half22float2(h);
        lo = f.x;
        hi = f.y;
      }
      const double a = (double)lo - c, b = (double)hi - c;
      s1 += a + b;
      s2 = fma(a, a, fma(b, b, s2));
    }
  }
}

// The shift: fp32 mean of the first min(n, 32) entries (one warp, fixed order;
// every caller gets the same value).
__device__ __forceinline__ float moments_shift(const void* K, int dtype, int64_t n, int lane) {
  const int k = n < 32 ? (int)n : 32;
  float x = lane < k ? load_f(K, lane, dtype) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x / (float)k;
}

__global__ void __launch_bounds__(kMomThreads) k_key_moments(const void* K, int dtype, int64_t n,
                                                            double* part) {
  __shared__ float s_c;
  pdl_launch_dependents();      // the merge kernel may launch; it waits for this grid
  if (threadIdx.x < 32) {
    const float c = moments_shift(K, dtype, n, threadIdx.x);
    if (threadIdx.x == 0) s_c = c;
  }
  __syncthreads();
  const double c = (double)s_c;
  const int per = dtype == TQ_F32 ? 4 : 8;              // entries per 16-byte load
  const int64_t nv = n / per;
  const int64_t nth = (int64_t)gridDim.x * kMomThreads;
  const int64_t t0 = (int64_t)blockIdx.x * kMomThreads + threadIdx.x;
  const uint4* v = static_cast<const uint4*>(K);
  double d1 = 0.0, d2 = 0.0;
  for (int64_t i = t0; i < nv; i += kMomUnroll * nth) {
    uint4 u[kMomUnroll];
#pragma unroll
    for (int k = 0; k < kMomUnroll; ++k)
      if (i + k * nth < nv) u[k] = __ldg(v + i + k * nth);
#pragma unroll
    for (int k = 0; k < kMomUnroll; ++k)
      if (i + k * nth < nv) moments16(u[k], dtype, c, d1, d2);
  }
  for (int64_t i = nv * per + t0; i < n; i += nth) {     // ragged tail
    const double x = (double)load_f(K, i, dtype) - c;
    d1 += x;
    d2 += x * x;
  }
  // fixed-order block reduction
  __shared__ double s_a[kMomThreads / 32], s_b[kMomThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    d1 += __shfl_xor_sync(0xffffffffu, d1, o);
    d2 += __shfl_xor_sync(0xffffffffu, d2, o);
  }
  if (lane == 0) {
    s_a[warp] = d1;
    s_b[warp] = d2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < kMomThreads / 32; ++w) {
      a += s_a[w];
      b += s_b[w];
    }
    part[2 * blockIdx.x] = a;
    part[2 * blockIdx.x + 1] = b;
  }
}

// out[0] = mean, out[1] = population variance (>= 0), from the blocks' shifted sums.
// Launched programmatically after k_key_moments: the shift (from K, which that
// kernel does not write) is formed before the wait for its partial sums.
__global__ void k_moments_final(const void* K, int dtype, int64_t n, const double* part, int nb,
                                double* out) {
  const int lane = threadIdx.x;
  const float c = moments_shift(K, dtype, n, lane);
  pdl_wait();
  double a = 0.0, b = 0.0;
  for (int i = lane; i < nb; i += 32) {
    a += part[2 * i];
    b += part[2 * i + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (lane == 0) {
    const double dn = (double)n, m1 = a / dn;
    const double var = b / dn - m1 * m1;
    out[0] = (double)c + m1;
    out[1] = var > 0.0 ? var : 0.0;
  }
}

double seq_mean(const double* x, int a, int b) {
  double t = 0.0;
  for (int i = a; i < b; ++i) t += x[i];
  return t / (double)(b - a);
}

double seq_sse(const double* x, int a, int b) {
  const double mu = seq_mean(x, a, b);
  double t = 0.0;
  for (int i = a; i < b; ++i) t += (x[i] - mu) * (x[i] - mu);
  return t;
}

}  // namespace

size_t key_moments_ws_bytes() { return (size_t)kMomBlocks * 2 * sizeof(double); }

cudaError_t launch_key_moments(const void* K, int dtype, int64_t n, double* out, double* part,
                               cudaStream_t s) {
  const int per = dtype == TQ_F32 ? 4 : 8;
  const int64_t nv = n / per;
  int64_t nb = (nv + (int64_t)kMomThreads * kMomUnroll - 1) / ((int64_t)kMomThreads * kMomUnroll);
  nb = nb < 1 ? 1 : (nb > kMomBlocks ? kMomBlocks : nb);
  k_key_moments<<<(unsigned)nb, kMomThreads, 0, s>>>(K, dtype, n, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_pdl(k_moments_final, dim3(1), dim3(32), 0, s, K, dtype, n,
                    static_cast<const double*>(part), (int)nb, out);
}

void sensitivity_segment(const double* var, int L, int k, int* bounds) {
  const double inf = INFINITY;
  // cost[g][l], with the boundary list of that optimum (g - 1 entries)
  std::vector<std::vector<double>> cost(k + 1, std::vector<double>(L + 1, inf));
  std::vector<std::vector<std::vector<int>>> bl(k + 1, std::vector<std::vector<int>>(L + 1));
  std::vector<std::vector<char>> have(k + 1, std::vector<char>(L + 1, 0));
  cost[0][0] = 0.0;
  have[0][0] = 1;
  for (int g = 1; g <= k; ++g) {
    for (int l = g; l <= L; ++l) {
      double best = inf;
      std::vector<int> bb;
      bool found = false;
      for (int a = g - 1; a < l; ++a) {
        if (!have[g - 1][a]) continue;
        const double c = cost[g - 1][a] + seq_sse(var, a, l);
        std::vector<int> cand = bl[g - 1][a];
        if (g > 1) cand.push_back(a);
        if (!found || c < best || (c == best && cand < bb)) {
          best = c;
          bb = cand;
          found = true;
        }
      }
      if (found) {
        cost[g][l] = best;
        bl[g][l] = bb;
        have[g][l] = 1;
      }
    }
  }
  for (int i = 0; i < k - 1; ++i) bounds[i] = bl[k][L][i];
}

int sensitivity_allocate(const double* var, int L, const int* bounds, int k, int m_avg, int m_min,
                         int m_max, int* m) {
  std::vector<int> edge(k + 1);
  edge[0] = 0;
  for (int i = 0; i < k - 1; ++i) edge[i + 1] = bounds[i];
  edge[k] = L;
  std::vector<int64_t> n(k);
  std::vector<double> s(k);
  int64_t left = (int64_t)L * m_avg;
  for (int g = 0; g < k; ++g) {
    n[g] = edge[g + 1] - edge[g];
    s[g] = seq_mean(var, edge[g], edge[g + 1]);
    m[g] = m_min;
    left -= n[g] * m_min;
  }
  if (left < 0) return -1;
  for (;;) {
    int pick = -1;
    double gain = 0.0;
    for (int g = 0; g < k; ++g) {
      if (m[g] + 32 > m_max || n[g] * 32 > left) continue;
      const double d = (double)n[g] * s[g] * (1.0 / m[g] - 1.0 / (m[g] + 32)) / (double)(n[g] * 32);
      if (d > gain) {
        pick = g;
        gain = d;
      }
    }
    if (pick < 0) return 0;
    m[pick] += 32;
    left -= n[pick] * 32;
  }
}

}  // namespace tq
