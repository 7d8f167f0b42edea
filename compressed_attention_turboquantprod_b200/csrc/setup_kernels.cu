// Setup kernels: Lloyd-Max codebook, Philox Gaussian fill, Householder QR -> Pi,
// and the sketch in rotated coordinates T = S Pi^T.  All float64, run once per
// (d, bits) or per layer; none of them is on the decode path.
#include <cmath>

#include "common.cuh"

namespace tq {
namespace {

// ---------------------------------------------------------------------------
// Lloyd-Max codebook ([TQ] 二: continuous 1-D k-means for the rotated-coordinate
// law f(t) ~ (1 - t^2)^((d-3)/2) on [-1, 1]).
//
// Interval mass: with t = sin(theta), (1 - t^2)^p dt = cos(theta)^(d-2) dtheta,
// an entire function of theta, integrated by composite 16-point Gauss-Legendre
// over 16 panels per cell; theta is clipped to +-min(pi/2, 14/sqrt(d-2)), where
// cos^(d-2) has fallen below e^-98 of its peak.  Partial first moment in closed
// form: int_a^b t (1 - t^2)^p dt = [(1-a^2)^(p+1) - (1-b^2)^(p+1)] / (2(p+1)).
// The normalising constant cancels in the centroid (moment / mass).
// ---------------------------------------------------------------------------
constexpr int kGL = 16;       // Gauss-Legendre nodes per panel
constexpr int kPanels = 16;   // panels per cell
constexpr int kMaxIter = 100000;

__device__ double pow_one_minus_sq(double t, double e) {   // (1 - t^2)^e, e > 0
  if (fabs(t) >= 1.0) return 0.0;
  return exp(e * log1p(-t * t));
}

__global__ void __launch_bounds__(256) k_codebook(int d, int bits, float* cent, float* bnd) {
  __shared__ double s_x[kGL], s_w[kGL];
  __shared__ double s_c[kMaxLevels], s_edge[kMaxLevels + 1];
  __shared__ double s_part[kMaxLevels][kPanels];
  __shared__ int s_done;
  const int tid = threadIdx.x;
  const int L = 1 << bits;

  // Gauss-Legendre nodes/weights on [-1, 1]: Newton on P_n from cos guesses.
  if (tid < kGL) {
    const int n = kGL;
    double x = cos(M_PI * (tid + 0.75) / (n + 0.5));
    double dp = 1.0;
    for (int it = 0; it < 100; ++it) {
      double p0 = 1.0, p1 = x;
      for (int k = 2; k <= n; ++k) {
        double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      dp = n * (x * p1 - p0) / (x * x - 1.0);
      double dx = p1 / dp;
      x -= dx;
      if (fabs(dx) < 1e-16) break;
    }
    // final derivative at the converged root
    double p0 = 1.0, p1 = x;
    for (int k = 2; k <= n; ++k) {
      double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
      p0 = p1;
      p1 = p2;
    }
    dp = n * (x * p1 - p0) / (x * x - 1.0);
    s_x[tid] = x;
    s_w[tid] = 2.0 / ((1.0 - x * x) * dp * dp);
  }
  if (tid < L) s_c[tid] = normcdfinv((tid + 0.5) / L) / sqrt((double)d);
  if (tid == 0) s_done = 0;
  __syncthreads();

  const double pm = 0.5 * (d - 1);           // p + 1
  const double theta_max = fmin(M_PI / 2, 14.0 / sqrt((double)(d - 2)));
  const int k = tid / kPanels, q = tid % kPanels;
  int iter = 0;
  for (iter = 1; iter <= kMaxIter; ++iter) {
    if (tid <= L) {
      s_edge[tid] = (tid == 0) ? -1.0 : (tid == L) ? 1.0 : 0.5 * (s_c[tid - 1] + s_c[tid]);
    }
    __syncthreads();
    if (k < L) {
      double a = fmax(asin(s_edge[k]), -theta_max);
      double b = fmin(asin(s_edge[k + 1]), theta_max);
      double sum = 0.0;
      if (b > a) {
        double h = (b - a) / kPanels;
        double lo = a + q * h;
        for (int i = 0; i < kGL; ++i) {
          double th = lo + 0.5 * h * (1.0 + s_x[i]);
          sum += s_w[i] * exp((d - 2) * log(cos(th)));
        }
        sum *= 0.5 * h;
      }
      s_part[k][q] = sum;
    }
    __syncthreads();
    if (tid == 0) {
      double delta = 0.0, cmax = 0.0;
      double cnew[kMaxLevels];
      for (int j = 0; j < L; ++j) {
        double mass = 0.0;
        for (int p = 0; p < kPanels; ++p) mass += s_part[j][p];
        double mom = (pow_one_minus_sq(s_edge[j], pm) - pow_one_minus_sq(s_edge[j + 1], pm)) /
                     (2.0 * pm);
        cnew[j] = mom / mass;
        delta = fmax(delta, fabs(cnew[j] - s_c[j]));
        cmax = fmax(cmax, fabs(cnew[j]));
      }
      for (int j = 0; j < L; ++j) s_c[j] = cnew[j];
      s_done = (delta < 1e-13 * cmax) ? 1 : 0;
    }
    __syncthreads();
    if (s_done) break;
  }
  if (tid == 0) {
    // exact antisymmetry, then fp32 storage rounding
    double c[kMaxLevels];
    const int half = L / 2;
    for (int j = 0; j < half; ++j) {
      double pos = 0.5 * (s_c[half + j] - s_c[half - 1 - j]);
      c[half + j] = pos;
      c[half - 1 - j] = -pos;
    }
    for (int j = 0; j < L; ++j) cent[j] = (float)c[j];
    for (int j = 0; j + 1 < L; ++j) bnd[j] = (j == half - 1) ? 0.0f : (float)(0.5 * (c[j] + c[j + 1]));
    if (!s_done) cent[0] = __int_as_float(0x7fc00000);   // NaN marks non-convergence
  }
}

// ---------------------------------------------------------------------------
// Philox4x64-10 (Salmon et al., SC'11) and the Box-Muller Gaussian.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void philox4x64_10(uint64_t c[4], uint64_t k0, uint64_t k1) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint64_t lo0 = M0 * c[0], hi0 = __umul64hi(M0, c[0]);
    const uint64_t lo1 = M1 * c[2], hi1 = __umul64hi(M1, c[2]);
    const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

__device__ __forceinline__ double gaussian_draw(uint64_t k, uint64_t seed, uint64_t stream) {
  uint64_t c[4] = {k, 0ull, 0ull, 0ull};
  philox4x64_10(c, seed, stream);
  const double u0 = ((double)(c[0] >> 11) + 0.5) * 0x1p-53;
  const double u1 = ((double)(c[1] >> 11) + 0.5) * 0x1p-53;
  return sqrt(-2.0 * log(u0)) * cos(6.283185307179586 * u1);
}

// Row-major rows x cols Gaussian matrix: into G64 (column-major) and/or S32 (row-major).
__global__ void k_gauss(double* G64, float* S32, int rows, int cols, uint64_t seed,
                        uint64_t stream) {
  const int64_t n = (int64_t)rows * cols;
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const double z = gaussian_draw((uint64_t)k, seed, stream);
  const int i = (int)(k / cols), j = (int)(k % cols);
  if (G64) G64[(int64_t)j * rows + i] = z;
  if (S32) S32[k] = (float)z;
}

// ---------------------------------------------------------------------------
// Householder QR of the d x d matrix A (column-major, float64) in place, then
// Q formed by backward accumulation, then Pi = Q diag(sign(diag R)) as fp32
// row-major.  One CTA; warps own columns, lanes run down rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_qr(double* A, double* Q, int d, float* Pi) {
  __shared__ double s_v[256];
  __shared__ double s_tau[256];
  __shared__ double s_sign[256];
  __shared__ double s_red[32];
  __shared__ double s_scale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  for (int k = 0; k < d; ++k) {
    double* colk = A + (int64_t)k * d;
    double ss = 0.0;
    for (int i = k + tid; i < d; i += blockDim.x) ss += colk[i] * colk[i];
    ss = warp_sum_d(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < nw; ++w) t += s_red[w];
      const double alpha = colk[k];
      const double sigma = sqrt(t);
      double beta, tau, scale;
      if (sigma == 0.0) {
        beta = alpha;
        tau = 0.0;
        scale = 0.0;
      } else {
        beta = alpha >= 0.0 ? -sigma : sigma;   // -sign(alpha) ||x||
        tau = (beta - alpha) / beta;
        scale = 1.0 / (alpha - beta);
      }
      s_scale = scale;
      s_tau[k] = tau;
      s_sign[k] = beta >= 0.0 ? 1.0 : -1.0;
      colk[k] = beta;
    }
    __syncthreads();
    const double scale = s_scale;
    for (int i = k + tid; i < d; i += blockDim.x) {
      const double v = (i == k) ? 1.0 : colk[i] * scale;
      s_v[i] = v;
      if (i > k) colk[i] = v;
    }
    __syncthreads();
    const double tau = s_tau[k];
    for (int j = k + 1 + warp; j < d; j += nw) {
      double* cj = A + (int64_t)j * d;
      double w = 0.0;
      for (int i = k + lane; i < d; i += 32) w += s_v[i] * cj[i];
      w = warp_sum_d(w) * tau;
      for (int i = k + lane; i < d; i += 32) cj[i] -= w * s_v[i];
    }
    __syncthreads();
  }
  for (int idx = tid; idx < d * d; idx += blockDim.x) Q[idx] = (idx / d == idx % d) ? 1.0 : 0.0;
  __syncthreads();
  for (int k = d - 1; k >= 0; --k) {
    for (int i = k + tid; i < d; i += blockDim.x) s_v[i] = (i == k) ? 1.0 : A[(int64_t)k * d + i];
    __syncthreads();
    const double tau = s_tau[k];
    for (int j = k + warp; j < d; j += nw) {
      double* qj = Q + (int64_t)j * d;
      double w = 0.0;
      for (int i = k + lane; i < d; i += 32) w += s_v[i] * qj[i];
      w = warp_sum_d(w) * tau;
      for (int i = k + lane; i < d; i += 32) qj[i] -= w * s_v[i];
    }
    __syncthreads();
  }
  for (int idx = tid; idx < d * d; idx += blockDim.x) {
    const int i = idx / d, j = idx % d;
    Pi[idx] = (float)(Q[(int64_t)j * d + i] * s_sign[j]);
  }
}

// Structured rotation Pi = H diag(s) / sqrt(d) ([NQ] six-stage pipeline, step 4:
// a Hadamard rotation): H[r][c] = (-1)^popcount(r & c) (Sylvester, d a power of
// two), s_c = +1 when the top bit of word 0 of Philox draw c (stream 2) is 0.
// Every entry is +-fl(1/sqrt(d)) (the reciprocal square root taken in float64).
__global__ void k_hadamard(float* Pi, int d, uint64_t seed) {
  const int64_t n = (int64_t)d * d;
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const int r = (int)(k / d), c = (int)(k % d);
  uint64_t w[4] = {(uint64_t)c, 0ull, 0ull, 0ull};
  philox4x64_10(w, seed, 2ull);
  const float mag = (float)(1.0 / sqrt((double)d));
  const bool neg = ((__popc((unsigned)(r & c)) & 1) != 0) != ((w[0] >> 63) != 0);
  Pi[k] = neg ? -mag : mag;
}

// T = S Pi^T (m x d), float64 accumulation of the stored fp32 values.
__global__ void k_sketch_rot(const float* S, const float* Pi, float* T, int m, int d) {
  const int a = blockIdx.x;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += (double)S[(int64_t)a * d + i] * (double)Pi[(int64_t)j * d + i];
    T[(int64_t)a * d + j] = (float)acc;
  }
}

}  // namespace

cudaError_t launch_projections_hadamard(int d, int m, uint64_t seed, float* Pi, float* S, float* T,
                                       cudaStream_t s) {
  const int threads = 256;
  {
    const int64_t n = (int64_t)m * d;
    k_gauss<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(nullptr, S, m, d, seed, 1);
  }
  {
    const int64_t n = (int64_t)d * d;
    k_hadamard<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(Pi, d, seed);
  }
  if (T) k_sketch_rot<<<m, 256, 0, s>>>(S, Pi, T, m, d);
  return cudaGetLastError();
}

cudaError_t launch_codebook(int d, int bits, float* cent, float* bnd, cudaStream_t s) {
  k_codebook<<<1, 256, 0, s>>>(d, bits, cent, bnd);
  return cudaGetLastError();
}

cudaError_t launch_projections(int d, int m, uint64_t seed, float* Pi, float* S, float* T,
                               double* ws, cudaStream_t s) {
  const int threads = 256;
  {
    const int64_t n = (int64_t)m * d;
    k_gauss<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(nullptr, S, m, d, seed, 1);
  }
  if (Pi) {
    double* A = ws;
    double* Q = ws + (int64_t)d * d;
    const int64_t n = (int64_t)d * d;
    k_gauss<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(A, nullptr, d, d, seed, 0);
    k_qr<<<1, 1024, 0, s>>>(A, Q, d, Pi);
    if (T) k_sketch_rot<<<m, 256, 0, s>>>(S, Pi, T, m, d);
  } else if (T) {
    cudaError_t e = cudaMemcpyAsync(T, S, sizeof(float) * (size_t)m * d, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace tq
