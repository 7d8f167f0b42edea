// Tensor-core decode attention for head dim 256 ([TQ] 四-六): G = 4 query heads
// per KV head, b1 <= 3 Lloyd-Max bits, m in {128, 256}, 4-bit values in groups
// of 64 (the long-context wide-head shape).
//
// The arithmetic is that of decode_mma.cu (int8 MMA logits on the stored bits
// with the query weights as four int8 slices; f16 MMA P V with the codes as f16
// subnormals and p * s split into f16 hi + lo), with three changes:
//  * b1 = 3: a symmetric 8-level codebook has four odd Walsh subsets {0}, {1},
//    {2}, {0,1,2}; the fourth feature plane is the XOR of the three stored
//    planes, formed on the fly (one LOP3 per 32 coordinates).
//  * 4-bit codes: a 16-bit half of a token-pair record holds 4 codes of each of
//    the two tokens; an AND of the word (shifted by a byte for the upper two)
//    keeps code k in {0, 1} of a byte of both, code * 16^k * 2^-24 as an f16
//    subnormal (the power of sixteen is undone at the end).
//  * 256 output channels need 64 accumulator registers per lane, so the two
//    warps of a pair work on the same block: each scores 32 of its 64 tokens,
//    the pair exchanges block maxima and probabilities through shared memory
//    (two pair barriers per block, double-buffered), and each warp accumulates
//    P V for 128 of the 256 channels over all 64 tokens.  Both warps of a pair
//    take identical running-max decisions, so their partial sums merge exactly.
// The two pairs of a CTA take alternate blocks; 2 CTAs are resident per SM.
#include <cfloat>

#include "mma_common.cuh"

namespace tq {
namespace mmadec {
namespace {

constexpr int WD = 256;          // head dim
constexpr int WNST = 4;          // stages: two per warp pair
constexpr int WT = 128;          // threads per CTA (2 pairs of 2 warps)
constexpr int WCTAS = 2;         // resident CTAs per SM (shared memory)
constexpr int kWPairBytes = 2 * WD * 4 / 8;   // value codes of a token pair (4-bit)

// s0 + 2^8 s1 + 2^16 s2 + 2^24 s3 with every slice sum below 2^24: each converts
// exactly; the result carries fp32 rounding only.
__device__ __forceinline__ float slices_to_float_wide(int s0, int s1, int s2, int s3) {
  return fmaf(16777216.f, __int2float_rn(s3),
              fmaf(65536.f, __int2float_rn(s2), fmaf(256.f, __int2float_rn(s1), __int2float_rn(s0))));
}

__device__ __forceinline__ void pair_sync(int pair) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
}

template <int B1, int KSQ>
__global__ void __launch_bounds__(WT, WCTAS) k_decode_partial_wide(MParams p) {
  constexpr int FS = B1;                             // stored bit-planes
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;      // feature planes (odd Walsh subsets)
  constexpr int NW = WD / 32;                        // words per plane per token
  constexpr int KSM = F * NW;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[WNST];
  __shared__ __align__(8) uint64_t ringbar;
  __shared__ int s_abort, s_abort_pair[2][2];       // [pair][buf]
  __shared__ int s_iss[WNST];
  __shared__ float s_bmax[2][2][2][MG];              // [pair][buf][half][head]
  __shared__ float s_p[2][2][64][MG];                // [pair][buf][token][head]
  __shared__ float s_m[2][MG], s_l[2][2][MG], s_mn[2][2][MG][4];
  __shared__ __align__(16) float s_qf[MG * WD];

  const Geom& g = p.g;
  const int split = blockIdx.x, unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int pair = warp >> 1, half = warp & 1;
  const int bq0 = b * p.Hq + h * MG;
  const int bb = (int)g.block_bytes;
  unsigned char* stage = smem_raw;                                            // [WNST][bb]
  float* s_out = reinterpret_cast<float*>(smem_raw + (size_t)WNST * bb);      // [2][MG][WD]

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
  const uint8_t* region = p.base + (int64_t)unit * g.region_bytes;

  // Ring tokens: the last split folds them in, a chunk of RC at a time staged in
  // the (until the final merge unused) s_out area; the first chunk is requested
  // at kernel start.
  const bool ring_split = split == p.splits - 1 && p.n_ring > 0;
  const int es = g.dtype == TQ_F32 ? 4 : 2;
  const int RC = (2 * MG * WD * (int)sizeof(float)) / (2 * WD * es);
  const unsigned char* ring_k = p.base + g.ring_k_off + (int64_t)unit * g.W * WD * es;
  const unsigned char* ring_v = p.base + g.ring_v_off + (int64_t)unit * g.W * WD * es;
  unsigned char* s_rk = reinterpret_cast<unsigned char*>(s_out);
  unsigned char* s_rv = s_rk + (size_t)RC * WD * es;

  if (tid == 0) {
    s_abort = 0;
    s_abort_pair[0][0] = s_abort_pair[0][1] = s_abort_pair[1][0] = s_abort_pair[1][1] = 0;
    for (int s = 0; s < WNST; ++s) mbar_init(&full[s], 1);
    mbar_init(&ringbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // launched programmatically after the preparation kernel (or the fused quantise
  // and preparation of a decode step): of what that grid may write, only the packed
  // blocks below p.early_blk are touched before the wait for it
  if (tid == 0) {
    for (int s = 0; s < WNST; ++s) s_iss[s] = 0;
    for (int s = 0; s < WNST && s < nb && blk0 + s < p.early_blk; ++s) {
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s], p.base, g.total_bytes, 209);
      s_iss[s] = 1;
    }
  }
  pdl_wait();
  if (tid == 0) {
    if (ring_split) {
      const uint32_t nbytes = (uint32_t)(min(RC, p.n_ring) * WD * es);
      mbar_expect_tx(&ringbar, 2 * nbytes);
      cache_bulk_load(s_rk, ring_k, nbytes, &ringbar, p.base, g.total_bytes, 202);
      cache_bulk_load(s_rv, ring_v, nbytes, &ringbar, p.base, g.total_bytes, 203);
    }
    for (int s = 0; s < WNST && s < nb; ++s) {
      if (s_iss[s]) continue;
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s], p.base, g.total_bytes, 204);
      s_iss[s] = 1;
    }
  }
  if (ring_split)
    for (int i = tid; i < MG * WD; i += WT) s_qf[i] = p.ws.qf[(int64_t)bq0 * WD + i];
  const uint4* fr = reinterpret_cast<const uint4*>(p.ws.frag + (int64_t)unit * ((KSM + KSQ) * 128)) + lane;
  const float* qc = p.ws.qconst + ((int64_t)unit * MG + tig) * 4;
  const float kM = qc[0], CM = qc[1], kQ = qc[2], CQ = qc[3];
  __syncthreads();

  const uint32_t maskA = 0x01010101u << tig, maskB = 0x10101010u << tig;
  // P V rows: row gid (h = 0) and gid + 8 (h = 1) of channel m-tile mt (0..7) of
  // this warp's half are channel 64 G + 4 gid + 32 ((mt >> 1) & 1) + 2 (mt & 1) + h
  // of value group G = 2 half + (mt >> 2): code 2 (mt & 1) + h of the 16-bit half
  // s = gid + 8 ((mt >> 1) & 1) of group G, i.e. word s * 4 + G of a token-pair
  // record, shifted right by 8 (mt & 1) and masked with 0x000F000F << 4h.

  float m_run = -INFINITY, l_run = 0.f;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
  float mnacc[4] = {0.f, 0.f, 0.f, 0.f};
  const float oddf = (gid & 1) ? 1.f : 0.f;
  const int hP = gid >> 1;
  constexpr float kLazy = 4.f;
  // raise the running max of head tig to m_new (the same value in both warps of
  // the pair), rescaling the running sum and the accumulators
  auto raise_to = [&](float bm) {
    const float m_new = fmaxf(m_run, bm);
    const float alpha = (m_run == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f) : exp2f(m_run - m_new);
    m_run = m_new;
    l_run *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][c] *= alpha;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) mnacc[gi] *= alpha;
  };
  auto warp_head_max = [&](float v) {
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
  };

  const int tb = 32 * half;
  for (int j = pair; j < nb; j += 2) {
    const int st = j % WNST;
    const int buf = (j >> 1) & 1;
    const uint32_t phase = (uint32_t)((j / WNST) & 1);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], phase));
    if (!ok && lane == 0) {
      atomicExch(p.err, 1);
      s_abort_pair[pair][buf] = 1;
      s_abort = 1;
    }
    const unsigned char* blk = stage + (size_t)st * bb;
    const int64_t tok0 = (blk0 + j) * kBlockTokens;
    const int nt_valid = (int)min((int64_t)kBlockTokens, p.n_comp - tok0);

    // ---------------- logits of this warp's tokens tb + 16 r + gid + 8 e
    float l[2][2] = {{-INFINITY, -INFINITY}, {-INFINITY, -INFINITY}};
    if (ok) {
      float vM[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, vQ[2][2];
      if constexpr (KSM > 0) {
        int a[2][2][4] = {};
#pragma unroll
        for (int c = 0; c < NW; c += 2) {
          // words c, c+1 of every stored plane, for the four rows
          uint32_t w[FS][2][2][2];
#pragma unroll
          for (int pl = 0; pl < FS; ++pl)
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                lds_words<2>(blk + g.o_idx + (tb + 16 * r + gid + 8 * e) * (FS * NW * 4) + pl * NW * 4 + 4 * c,
                             w[pl][r][e]);
#pragma unroll
          for (int f = 0; f < F; ++f)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const uint4 bq = __ldg(fr + (f * NW + c + kk) * 32);
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                uint32_t x0, x1;
                if (f < FS) {
                  x0 = w[f][r][0][kk];
                  x1 = w[f][r][1][kk];
                } else {      // f == 3: the parity of the three stored planes
                  x0 = w[0][r][0][kk] ^ w[FS > 1 ? 1 : 0][r][0][kk] ^ w[FS > 2 ? 2 : 0][r][0][kk];
                  x1 = w[0][r][1][kk] ^ w[FS > 1 ? 1 : 0][r][1][kk] ^ w[FS > 2 ? 2 : 0][r][1][kk];
                }
                imma16832(a[r][0], x0 & maskA, x1 & maskA, x0 & maskB, x1 & maskB, bq.x, bq.y);
                imma16832(a[r][1], x0 & maskA, x1 & maskA, x0 & maskB, x1 & maskB, bq.z, bq.w);
              }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            vM[r][e] = slices_to_float_wide(a[r][0][2 * e], a[r][0][2 * e + 1], a[r][1][2 * e],
                                            a[r][1][2 * e + 1]);
      }
      {
        int a[2][2][4] = {};
#pragma unroll
        for (int c = 0; c < KSQ; c += 4) {
          uint32_t w[2][2][4];
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              lds_words<4>(blk + g.o_sign + (tb + 16 * r + gid + 8 * e) * (KSQ * 4) + 4 * c, w[r][e]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint4 bq = __ldg(fr + (KSM + c + kk) * 32);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint32_t x0 = w[r][0][kk], x1 = w[r][1][kk];
              imma16832(a[r][0], x0 & maskA, x1 & maskA, x0 & maskB, x1 & maskB, bq.x, bq.y);
              imma16832(a[r][1], x0 & maskA, x1 & maskA, x0 & maskB, x1 & maskB, bq.z, bq.w);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            vQ[r][e] = slices_to_float_wide(a[r][0][2 * e], a[r][0][2 * e + 1], a[r][1][2 * e],
                                            a[r][1][2 * e + 1]);
      }
      const float* rho = reinterpret_cast<const float*>(blk + g.o_rho);
      const float* rn = reinterpret_cast<const float*>(blk + g.o_rnorm);
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = tb + 16 * r + gid + 8 * e;
          const float v = B1 > 0 ? rho[t] * fmaf(kM, vM[r][e], CM) + rn[t] * fmaf(kQ, vQ[r][e], CQ)
                                 : rho[t] * fmaf(kQ, vQ[r][e], CQ);
          l[r][e] = t < nt_valid ? v : -INFINITY;
        }
      if (p.logits) {
        const float inv = 1.f / p.scale_log2;
        float* lg = p.logits + (int64_t)(bq0 + tig) * p.n_log + tok0;
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int t = tb + 16 * r + gid + 8 * e;
            if (t < nt_valid) lg[t] = l[r][e] * inv;
          }
      }
    }

    // ---------------- block max of the pair, lazy running max, probabilities
    {
      const float lm = warp_head_max(fmaxf(fmaxf(l[0][0], l[0][1]), fmaxf(l[1][0], l[1][1])));
      if (gid == 0) s_bmax[pair][buf][half][tig] = lm;
    }
    pair_sync(pair);
    const float bm = fmaxf(s_bmax[pair][buf][0][tig], s_bmax[pair][buf][1][tig]);
    if (__any_sync(0xffffffffu, bm > m_run + kLazy)) raise_to(bm);
    {
      float pr[2][2];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) pr[r][e] = m_run == -INFINITY ? 0.f : exp2f(l[r][e] - m_run);
      l_run += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
      const float4* vm4 = reinterpret_cast<const float4*>(blk + g.o_vmin);
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = tb + 16 * r + gid + 8 * e;
          s_p[pair][buf][t][tig] = pr[r][e];
          if (ok) {
            const float4 mv = vm4[t];
            mnacc[0] = fmaf(pr[r][e], mv.x, mnacc[0]);
            mnacc[1] = fmaf(pr[r][e], mv.y, mnacc[1]);
            mnacc[2] = fmaf(pr[r][e], mv.z, mnacc[2]);
            mnacc[3] = fmaf(pr[r][e], mv.w, mnacc[3]);
          }
        }
    }
    pair_sync(pair);
    const bool pair_ok = s_abort_pair[pair][buf] == 0;

    // ---------------- P V of all 64 tokens on channels 128 half .. +127
    if (pair_ok) {
#pragma unroll 1
      for (int tm = 0; tm < 4; ++tm) {
        // MMA indices k = 2tig, 2tig+1 are the m-tile's tokens TA = 2tig, TB = TA+1
        // (token pair tig), k = 2tig+8, 2tig+9 are TC = TA+8, TD = TA+9 (pair tig+4)
        const int TA = 16 * tm + 2 * tig, TB = TA + 1, TC = TA + 8, TD = TA + 9;
        const float pA = s_p[pair][buf][TA][hP], pB = s_p[pair][buf][TB][hP];
        const float pC = s_p[pair][buf][TC][hP], pD = s_p[pair][buf][TD][hP];
        const float* vs = reinterpret_cast<const float*>(blk + g.o_vscale);
        const float2 sA = *reinterpret_cast<const float2*>(vs + 4 * TA + 2 * half);
        const float2 sB = *reinterpret_cast<const float2*>(vs + 4 * TB + 2 * half);
        const float2 sC = *reinterpret_cast<const float2*>(vs + 4 * TC + 2 * half);
        const float2 sD = *reinterpret_cast<const float2*>(vs + 4 * TD + 2 * half);
        uint32_t bpv[2][2];
        {
          const float sa[2] = {sA.x, sA.y}, sb[2] = {sB.x, sB.y};
          const float sc[2] = {sC.x, sC.y}, sd[2] = {sD.x, sD.y};
          const float2 pAB = make_float2(pA, pB), pCD = make_float2(pC, pD);
          const float2 nodd = make_float2(-oddf, -oddf);
#pragma unroll
          for (int gi = 0; gi < 2; ++gi) {
            const float2 x0 = mul2(pAB, make_float2(sa[gi], sb[gi]));
            const float2 x1 = mul2(pCD, make_float2(sc[gi], sd[gi]));
            // column gid even carries fp16(x), odd carries fp16(x - fp16(x))
            const float2 f0 = __half22float2(__floats2half2_rn(x0.x, x0.y));
            const float2 f1 = __half22float2(__floats2half2_rn(x1.x, x1.y));
            const float2 l0 = fma2(nodd, f0, x0), l1 = fma2(nodd, f1, x1);
            __half2 h0 = __floats2half2_rn(l0.x, l0.y);
            __half2 h1 = __floats2half2_rn(l1.x, l1.y);
            bpv[gi][0] = *reinterpret_cast<uint32_t*>(&h0);
            bpv[gi][1] = *reinterpret_cast<uint32_t*>(&h1);
          }
        }
        // words (s, G) = (gid + 8 u, 2 half + v) of the pairs tig and tig + 4
        const unsigned char* vc = blk + g.o_vcode + 16 * gid + 8 * half;
        uint2 wAB[2], wCD[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          wAB[u] = *reinterpret_cast<const uint2*>(vc + (TA >> 1) * kWPairBytes + 128 * u);
          wCD[u] = *reinterpret_cast<const uint2*>(vc + (TC >> 1) * kWPairBytes + 128 * u);
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int u = (mt >> 1) & 1, v = mt >> 2, sh = 8 * (mt & 1);
          const uint32_t ab = (v ? wAB[u].y : wAB[u].x) >> sh, cd = (v ? wCD[u].y : wCD[u].x) >> sh;
          hmma16816(acc[mt], ab & 0x000F000Fu, ab & 0x00F000F0u, cd & 0x000F000Fu, cd & 0x00F000F0u,
                    bpv[v][0], bpv[v][1]);
        }
      }
    }
    // Release the stage: once both warps of the pair are past this barrier, the
    // pair's first warp refills it with block j + WNST (same parity, so the same
    // pair consumes it).
    pair_sync(pair);
    if (pair_ok && half == 0 && lane == 0 && j + WNST < nb && !s_abort) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&full[st], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)st * bb, region + (blk0 + j + WNST) * bb, (uint32_t)bb, &full[st], p.base, g.total_bytes, 205);
      s_iss[st] += 1;
    }
    if (!pair_ok) break;       // both warps of the pair read the same flag after the same barrier
  }
  __syncthreads();

  if (s_abort) {
    // a wait gave up: wait (bounded) for the last copy issued into every stage, then leave
    if (tid == 0) {
      for (int s = 0; s < WNST; ++s)
        if (s_iss[s] > 0) (void)mbar_wait(&full[s], (uint32_t)((s_iss[s] - 1) & 1));
      if (ring_split) (void)mbar_wait(&ringbar, 0);
    }
    return;
  }

  // acc[mt][c] is channel chan(mt) (+1 for c >= 2) of head tig in units of
  // 2^-24 (row gid + 8: 2^-20)
  auto chan = [&](int mt) {
    return 64 * (2 * half + (mt >> 2)) + 4 * gid + 32 * ((mt >> 1) & 1) + 2 * (mt & 1);
  };
  auto code_unit = [&](int mt) { return (void)mt, 5.9604644775390625e-8f; };   // 2^-24
  // ---------------- exact ring tokens (last split): pair q takes slots
  // per_pair q .. +per_pair-1 of each chunk; both warps of the pair score them
  // (identical logits, identical running-max decisions), each adds p v on its
  // channel half, and only half 0 counts p in the running sum.
  if (ring_split) {
    const int64_t first = p.n_total - p.n_ring;
    const int per_pair = RC / 2;
    for (int c0 = 0, ci = 0; c0 < p.n_ring; c0 += RC, ++ci) {
      const int nc = min(RC, p.n_ring - c0);
      if (ci > 0 && tid == 0) {
        const uint32_t nbytes = (uint32_t)(nc * WD * es);
        mbar_expect_tx(&ringbar, 2 * nbytes);
        cache_bulk_load(s_rk, ring_k + (int64_t)c0 * WD * es, nbytes, &ringbar, p.base, g.total_bytes, 206);
        cache_bulk_load(s_rv, ring_v + (int64_t)c0 * WD * es, nbytes, &ringbar, p.base, g.total_bytes, 207);
      }
      const bool rok = __all_sync(0xffffffffu, mbar_wait(&ringbar, (uint32_t)(ci & 1)));
      if (!rok && lane == 0) {
        atomicExch(p.err, 1);
        s_abort = 1;
      }
      __syncthreads();
      if (s_abort) {
        if (tid == 0) (void)mbar_wait(&ringbar, (uint32_t)(ci & 1));
        return;
      }
      const int sl = per_pair * pair + gid;
      float lr = -INFINITY;
      if (gid < per_pair && sl < nc) {
        const float* q = s_qf + tig * WD;
        float dot = 0.f;
#pragma unroll 8
        for (int jj = 0; jj < WD; ++jj) dot = fmaf(q[jj], load_f(s_rk, (int64_t)sl * WD + jj, g.dtype), dot);
        const int64_t rt = ((int64_t)(c0 + sl) - first % g.W + g.W) % g.W;
        if (p.logits && half == 0) p.logits[(int64_t)(bq0 + tig) * p.n_log + p.n_comp + rt] = dot;
        lr = dot * p.scale_log2;
      }
      const float lmax = warp_head_max(lr);
      if (__any_sync(0xffffffffu, lmax > m_run + kLazy)) raise_to(lmax);
      const float p0 = m_run == -INFINITY ? 0.f : exp2f(lr - m_run);
      if (half == 0) l_run += p0;
      for (int T = 0; T < per_pair; ++T) {
        const float pt = __shfl_sync(0xffffffffu, p0, 4 * T + tig);
        const int sl2 = per_pair * pair + T;
        if (sl2 >= nc) break;
        const int64_t e = (int64_t)sl2 * WD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const float v0 = load_f(s_rv, e + chan(mt), g.dtype);
          const float v1 = load_f(s_rv, e + chan(mt) + 1, g.dtype);
          const float u = code_unit(mt);
          acc[mt][0] = fmaf(pt * v0, u, acc[mt][0]);
          acc[mt][2] = fmaf(pt * v1, 16.f * u, acc[mt][2]);
        }
      }
      __syncthreads();     // the chunk is consumed before the next one is requested
    }
  }

  // ---------------- merge: the two warps of a pair share m; the pairs differ
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  if (gid == 0) {
    if (half == 0) s_m[pair][tig] = m_run;
    s_l[pair][half][tig] = l_run;
  }
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    float v = mnacc[gi];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    if (gid == 0) s_mn[pair][half][tig][gi] = v;
  }
  __syncthreads();
  const float Mh = fmaxf(s_m[0][tig], s_m[1][tig]);
  const float sc = (m_run == -INFINITY) ? 0.f : exp2f(m_run - Mh);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int grp = 2 * half + (mt >> 2);
    const float mnv = s_mn[pair][0][tig][grp] + s_mn[pair][1][tig][grp];
    const float inv = 16777216.f;      // 2^24 = 1 / code_unit(mt)
    *reinterpret_cast<float2*>(&s_out[(pair * MG + tig) * WD + chan(mt)]) =
        make_float2(((acc[mt][0] + acc[mt][1]) * inv + mnv) * sc,
                    ((acc[mt][2] + acc[mt][3]) * (0.0625f * inv) + mnv) * sc);
  }
  __syncthreads();
  for (int i = tid; i < MG * WD; i += WT) {
    const int hh = i / WD, ch = i % WD;
    p.ws.part_o[((int64_t)(bq0 + hh) * p.splits + split) * WD + ch] =
        s_out[hh * WD + ch] + s_out[(MG + hh) * WD + ch];
  }
  if (tid < MG) {
    const float M = fmaxf(s_m[0][tid], s_m[1][tid]);
    float L = 0.f;
    if (M != -INFINITY)
      for (int q = 0; q < 2; ++q)
        if (s_m[q][tid] != -INFINITY) L += (s_l[q][0][tid] + s_l[q][1][tid]) * exp2f(s_m[q][tid] - M);
    p.ws.part_ml[((int64_t)(bq0 + tid) * p.splits + split) * 2 + 0] = M;
    p.ws.part_ml[((int64_t)(bq0 + tid) * p.splits + split) * 2 + 1] = L;
  }
  if (!p.out) return;
  // The last split of this unit to finish merges all splits' (m, l, o).
  __shared__ int s_last;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int done = atomicAdd(&p.ws.counter[unit], 1);
    s_last = (done == p.splits - 1);
    if (s_last) p.ws.counter[unit] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (p.splits <= 32) {
    merge_splits<WD, WT>(p, bq0);
    return;
  }
  for (int i = tid; i < MG * WD; i += WT) {
    const int hh = i / WD, ch = i % WD;
    const int bq = bq0 + hh;
    const volatile float* ml = p.ws.part_ml + (int64_t)bq * p.splits * 2;
    const volatile float* po = p.ws.part_o + (int64_t)bq * p.splits * WD;
    float M = -INFINITY;
    for (int sp = 0; sp < p.splits; ++sp) M = fmaxf(M, ml[2 * sp]);
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int sp = 0; sp < p.splits; ++sp) {
        const float ms = ml[2 * sp];
        if (ms == -INFINITY) continue;
        const float wgt = exp2f(ms - M);
        L = fmaf(ml[2 * sp + 1], wgt, L);
        o = fmaf(po[sp * WD + ch], wgt, o);
      }
      o = o / L;
    }
    store_f(p.out, (int64_t)bq * WD + ch, g.dtype, o);
  }
}

template <int B1, int KSQ>
cudaError_t launch_wide_t(const MParams& p, cudaStream_t s) {
  const size_t smem = (size_t)WNST * p.g.block_bytes + sizeof(float) * 2 * MG * WD;
  cudaError_t e = cudaFuncSetAttribute(k_decode_partial_wide<B1, KSQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.splits, (unsigned)(p.g.B * p.g.Hkv));
  return launch_pdl(k_decode_partial_wide<B1, KSQ>, grid, dim3(WT), smem, s, p);
}

}  // namespace

bool decode_wide_supported(const Geom& g, int G) {
  return g.d == WD && G == MG && g.vbits == 4 && g.group == 64 && g.b1 <= 3 &&
         (g.m == 128 || g.m == 256);
}

cudaError_t launch_partial_wide(const MParams& p, cudaStream_t s) {
  switch (p.g.b1 * 32 + p.g.m / 32) {
    case 0 * 32 + 4: return launch_wide_t<0, 4>(p, s);
    case 0 * 32 + 8: return launch_wide_t<0, 8>(p, s);
    case 1 * 32 + 4: return launch_wide_t<1, 4>(p, s);
    case 1 * 32 + 8: return launch_wide_t<1, 8>(p, s);
    case 2 * 32 + 4: return launch_wide_t<2, 4>(p, s);
    case 2 * 32 + 8: return launch_wide_t<2, 8>(p, s);
    case 3 * 32 + 4: return launch_wide_t<3, 4>(p, s);
    case 3 * 32 + 8: return launch_wide_t<3, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mmadec

TQ_BOUNDS_READER(bounds_flag_wide)

}  // namespace tq
