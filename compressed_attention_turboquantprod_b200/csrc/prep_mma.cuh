// Query preparation of the tensor-core decode paths (one CTA of 256 threads per
// (batch, KV head)), shared by the preparation kernel (decode_mma.cu) and the
// fused append-and-prepare kernel of a decode step (quant_kernels.cu).
#pragma once

#include "mma_common.cuh"

namespace tq {
namespace mmadec {

// Dynamic shared memory of prep_mma_body: the queries, Pi q and S q of the G heads.
__host__ __device__ inline size_t prep_smem_bytes(int d, int m) { return sizeof(float) * MG * (2 * d + m); }

// ---------------------------------------------------------------- prep
// For the G = 4 queries of one (b, KV head):
//  * qf = q in fp32 (for the ring), qr = Pi q, qs = sqrt(pi/2)/m S q, each row of
//    [Pi; S] read once (a float4 per lane) and dotted with the four queries;
//  * the Walsh weights of the codebook, the 24-bit fixed-point quantisation of
//    the query weights and their four int8 slices laid out as the lanes' B
//    fragments, and the per-head affine constants of the logit (log2 units);
//  * zeroes the unit's split counter and, in unit 0, the error flag.
// The MSE half (rows of Pi, the plane fragments, constants kM / CM, qf and the
// counters) and the QJL half (rows of S, the sign fragments, kQ / CQ) need
// nothing from each other: part 0 does the first, part 1 the second, part 2
// both (one CTA of 256 threads per (unit, part)).
template <int NV>     // float4s of a row per lane: head dim 128 * NV
__device__ __forceinline__ void prep_mma_body(const Geom& g, const void* Q, int Hq, const float* Pi,
                                              const float* S, const float* cent, float scale_log2,
                                              const DecodeWs& ws, int unit, int part,
                                              unsigned char* smem_raw) {
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int d = g.d, m = g.m, b1 = g.b1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool do_mse = part != 1, do_qjl = part != 0;
  float* sq = reinterpret_cast<float*>(smem_raw);     // [G][d]
  float* sqr = sq + MG * d;                           // [G][d]
  float* sqs = sqr + MG * d;                          // [G][m]
  __shared__ float s_w[4];                            // Walsh weights of the odd subsets
  __shared__ float s_cent[8];
  __shared__ unsigned s_maxM[MG], s_maxQ[MG];
  __shared__ float s_sumqr[MG], s_sumqs[MG];
  const int bq0 = b * Hq + h * MG;
  const int rows_pi = b1 > 0 ? d : 0;
  // this part's rows of [Pi; S]: [r_begin, r_end) (with the structured rotation, Pi q
  // is a butterfly instead: no rows of Pi are read but row 0)
  const int r_begin = do_mse && !g.hadamard ? 0 : rows_pi, r_end = do_qjl ? rows_pi + m : rows_pi;
  {
    // the rows are read after the queries: start them towards L2 now
    const int l0 = r_begin * d / 32, l1 = r_end * d / 32, lines_pi = rows_pi * d / 32;
    for (int i = l0 + tid; i < l1; i += blockDim.x)
      prefetch_l2(i < lines_pi ? Pi + 32 * (int64_t)i : S + 32 * (int64_t)(i - lines_pi));
  }
  if (tid == 0 && do_mse) {
    ws.counter[unit] = 0;
    if (unit == 0) *ws.err = 0;
  }
  // the codebook and the queries are requested together
  const int L = b1 > 0 ? 1 << b1 : 0;
  if (tid < 8) s_cent[tid] = tid < L ? cent[tid] : 0.f;
  for (int i = tid; i < MG * d; i += blockDim.x) {
    const float v = load_f(Q, (int64_t)bq0 * d + i, g.dtype);
    sq[i] = v;
    if (do_mse) ws.qf[(int64_t)bq0 * d + i] = v;
  }
  __syncthreads();
  if (tid < 4) {
    // w_S = (1/L) sum_idx c[idx] (-1)^{popc(idx & S)} for the odd subsets S, in the
    // order of the feature planes: {0}, {1}, {2}, {0,1,2} (thread k: subset k).
    const int subset = tid < 3 ? 1 << tid : 7;
    double acc = 0.0;
    for (int idx = 0; idx < L; ++idx)
      acc += (double)s_cent[idx] * ((__popc(idx & subset) & 1) ? -1.0 : 1.0);
    s_w[tid] = L ? (float)(acc / L) : 0.f;
  }
  const float qscale = 1.2533141373155003f / (float)m;
  // Rows in passes of 8 per warp: lane l dots float4 l of each row (coalesced)
  // with columns 4l..4l+3 of the four queries (held in registers); a
  // reduce-scatter over the warp then leaves the sum of (row l/4, head l%4) in
  // lane l.  (NV float4s per lane per row: columns 128 c + 4 lane.)
  if (g.hadamard && do_mse && warp < MG) {   // Pi q = H (Pi[0,:] * q), head = warp
    warp_hadamard_rotate(Pi, sq + warp * d, 1.f, sqr + warp * d, d, lane);
    for (int j = lane; j < d; j += 32) ws.qr[(int64_t)(bq0 + warp) * d + j] = sqr[warp * d + j];
  }
  float4 qv[MG][NV];
#pragma unroll
  for (int hh = 0; hh < MG; ++hh)
#pragma unroll
    for (int c = 0; c < NV; ++c)
      qv[hh][c] = *reinterpret_cast<const float4*>(sq + hh * d + 128 * c + 4 * lane);
  for (int r0 = r_begin + 8 * warp; r0 < r_end; r0 += 8 * (blockDim.x / 32)) {
    float4 wv[8][NV];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = r0 + k;
      const float* row = r < rows_pi ? Pi + (int64_t)r * d : S + (int64_t)(r - rows_pi) * d;
#pragma unroll
      for (int c = 0; c < NV; ++c) wv[k][c] = *reinterpret_cast<const float4*>(row + 128 * c + 4 * lane);
    }
    float v[32];
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int hh = 0; hh < MG; ++hh) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < NV; ++c)
          a = fmaf(wv[k][c].x, qv[hh][c].x, fmaf(wv[k][c].y, qv[hh][c].y,
              fmaf(wv[k][c].z, qv[hh][c].z, fmaf(wv[k][c].w, qv[hh][c].w, a))));
        v[4 * k + hh] = a;
      }
    // reduce-scatter: after the round with offset o, a lane keeps the half of its
    // values selected by (lane & o) and adds its partner's copy of that half
#pragma unroll
    for (int o = 16, n = 16; o >= 1; o >>= 1, n >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int k = 0; k < n; ++k) {
        const float send = upper ? v[k] : v[k + n];
        const float keep = upper ? v[k + n] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const int r = r0 + (lane >> 2), hh = lane & 3;
    const float a = v[0];
    if (r < rows_pi) {
      sqr[hh * d + r] = a;
      ws.qr[(int64_t)(bq0 + hh) * d + r] = a;
    } else {
      sqs[hh * m + (r - rows_pi)] = a * qscale;
      ws.qs[(int64_t)(bq0 + hh) * m + (r - rows_pi)] = a * qscale;
    }
  }
  __syncthreads();
  const int F = b1 > 0 ? 1 << (b1 - 1) : 0;     // feature planes per coordinate
  {
    // warps 0-3: MSE weights of head w (max |W|, sum qr); warps 4-7: QJL of head w-4
    const int hh = warp & 3;
    float mx = 0.f, sm = 0.f;
    if (warp < 4) {
      float wk = 0.f;
      for (int k = 0; k < F; ++k) wk = fmaxf(wk, fabsf(2.f * s_w[k]));
      if (F && do_mse)
        for (int j = lane; j < d; j += 32) {
          const float qr = sqr[hh * d + j];
          mx = fmaxf(mx, wk * fabsf(qr));
          sm += qr;
        }
    } else if (do_qjl) {
      for (int i = lane; i < m; i += 32) {
        const float qs = sqs[hh * m + i];
        mx = fmaxf(mx, fabsf(2.f * qs));
        sm += qs;
      }
    }
    mx = warp_max(mx);
    sm = warp_sum(sm);
    if (lane == 0) {
      if (warp < 4) {
        s_maxM[hh] = __float_as_uint(mx);
        s_sumqr[hh] = sm;
      } else {
        s_maxQ[hh] = __float_as_uint(mx);
        s_sumqs[hh] = sm;
      }
    }
  }
  __syncthreads();
  // query weights in fixed point with |W| <= kFix = 2^24 - 2^17, so that W * 2^7
  // (the largest A-byte compensation) stays below 2^31 and splits into four
  // signed int8 slices
  const float kFix = 16646144.f;
  if (tid < MG) {
    const float mM = __uint_as_float(s_maxM[tid]), mQ = __uint_as_float(s_maxQ[tid]);
    float* c = ws.qconst + ((int64_t)unit * MG + tid) * 4;
    if (do_mse) {
      const float dM = mM > 0.f ? mM / kFix : 1.f;
      float wsum = 0.f;
      for (int k = 0; k < F; ++k) wsum += s_w[k];
      c[0] = dM / 128.f * scale_log2;
      c[1] = wsum * s_sumqr[tid] * scale_log2;
    }
    if (do_qjl) {
      const float dQ = mQ > 0.f ? mQ / kFix : 1.f;
      c[2] = dQ / 128.f * scale_log2;
      c[3] = -s_sumqs[tid] * scale_log2;
    }
  }
  const int ksM = F * d / 32, ksQ = m / 32;
  const int w0 = do_mse ? 0 : ksM * 128, w1 = do_qjl ? (ksM + ksQ) * 128 : ksM * 128;
  uint32_t* fr = ws.frag + (int64_t)unit * (ksM + ksQ) * 128;
  const int kpp = d / 32;                          // k-steps per feature plane
  for (int wi = w0 + tid; wi < w1; wi += blockDim.x) {
    // word order [ks][lane][ntile][reg]: a lane's four words of a k-step are one uint4
    const int r = wi & 1, nt = (wi >> 1) & 1, ln = (wi >> 2) & 31, ks = wi >> 7;
    const int col = ln >> 2, tg = ln & 3;
    const int hh = col >> 1;
    const int slice = 2 * nt + (col & 1);
    // the A byte of MMA index k carries 2^t (k < 16) or 2^(4+t) (k >= 16), t = tg
    const int shift = r ? 3 - tg : 7 - tg;
    uint32_t word = 0;
    {
      const bool mse = ks < ksM;
      const float mx = __uint_as_float(mse ? s_maxM[hh] : s_maxQ[hh]);
      const float inv_delta = mx > 0.f ? kFix / mx : 1.f;
      const int plane = mse ? ks / kpp : 0, jb = mse ? (ks - plane * kpp) * 32 : (ks - ksM) * 32;
      const float wsc = mse ? -2.f * s_w[plane] : 2.f;
      const float* src = mse ? sqr + hh * d + jb : sqs + hh * m + jb;
      for (int i = 0; i < 4; ++i) {
        const int bit = tg + 8 * i + (r ? 4 : 0);
        const float w = wsc * src[bit];
        const int wint = __float2int_rn(w * inv_delta) * (1 << shift);   // |wint| < 2^31
        const int s0 = ((wint + 128) & 255) - 128;
        const int t1 = (wint - s0) >> 8;
        const int s1 = ((t1 + 128) & 255) - 128;
        const int t2 = (t1 - s1) >> 8;
        const int s2 = ((t2 + 128) & 255) - 128;
        const int s3 = (t2 - s2) >> 8;
        const int sv = slice == 0 ? s0 : slice == 1 ? s1 : slice == 2 ? s2 : s3;
        word |= ((uint32_t)(sv & 255)) << (8 * i);
      }
    }
    fr[wi] = word;
  }
}

}  // namespace mmadec
}  // namespace tq
