// Multi-token (chunked prefill) attention on the packed cache: a chunk of n new
// tokens is scored against the compressed history ([TQ] 四-六 estimator, 2-bit
// value groups), the exact ring and, causally, the chunk itself, before the chunk
// is appended.
//
// The chunk's queries form a virtual batch of B * n decode queries (query token i
// of batch b is virtual batch b n + i), so the query preparation, the partial
// layout and the split merge are the decode's.  Two kernels here:
//
//   k_prefill_partial_mma  history partials on the tensor cores.  Same operands as
//       the decode (int8 score MMAs over the stored bit-planes with the query
//       weights as four int8 slices; f16 P V MMAs over the token-pair value
//       words), but every warp owns QG = 2 query tokens (2 x 4 heads) and walks
//       all 64 tokens of every staged block, so one masked key operand serves two
//       query tokens and one staged block serves up to 8 (4 warps).  Each warp's
//       softmax state covers all tokens of the split, so its (m, l, o) go straight
//       to the partial slots without a cross-warp merge.
//   k_prefill_exact        the exact segment of every query (ring + chunk tokens
//       0..i) on CUDA cores, written as one more partial slot.
//
// Specialisation of the tensor-core kernel: head dim 128, G = 4, 2-bit values in
// groups of 32, b1 in {0, 1, 2}, m in {64, ..., 512} (the decode's d = 128 path).
#include <cfloat>

#include "mma_common.cuh"

namespace tq {
namespace {
using namespace mmadec;

constexpr int MD = 128;
constexpr int QG = 2;            // query tokens per warp
#ifndef TQ_PREFILL_WARPS
#define TQ_PREFILL_WARPS 4
#endif
constexpr int PNW = TQ_PREFILL_WARPS;   // warps per CTA at most
constexpr int kPrefillRegs = 232;       // registers per thread of the partial kernel (bound)
constexpr int PNST = 4;          // staged blocks in flight
constexpr int kPairBytes = 2 * MD * 2 / 8;   // value codes of a token pair (2-bit)

struct PParams {
  Geom g;                 // the cache's geometry (batch B)
  const uint8_t* base;
  int64_t n_comp;         // compressed tokens
  int nq, Hq;             // chunk length, query heads
  int splits, nslots, bps;
  int q_per_cta;          // query tokens per CTA (QG x warps)
  DecodeWs ws;            // carved for the virtual batch B * nq
  int* err;
};

template <int B1, int KSQ>
__global__ void __launch_bounds__(PNW * 32, 1) k_prefill_partial_mma(PParams p) {
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;
  constexpr int KSM = F * MD / 32;
  constexpr int KS = KSM + KSQ;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[PNST];
  __shared__ int s_cnt[PNST], s_iss[PNST];
  __shared__ int s_abort;

  const Geom& g = p.g;
  const int qtile = blockIdx.x, split = blockIdx.y, unit = blockIdx.z;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int nw = blockDim.x >> 5;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int bb = (int)g.block_bytes;
  unsigned char* stage = smem_raw;                                                  // [PNST][bb]
  uint4* s_frag4 = reinterpret_cast<uint4*>(smem_raw + (size_t)PNST * bb);         // [nw*QG][KS][32]

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
  const uint8_t* region = p.base + (int64_t)unit * g.region_bytes;

  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < PNST; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // launched programmatically after the preparation kernel
  pdl_wait();
  if (tid == 0) {
    for (int s = 0; s < PNST; ++s) s_iss[s] = 0;
    for (int s = 0; s < PNST && s < nb; ++s) {
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s], p.base, g.total_bytes, 302);
      s_iss[s] = 1;
    }
  }
  if (tid < PNST) s_cnt[tid] = 0;

  // this warp's query tokens (a token past the chunk end repeats the last one and
  // is not written)
  int qi[QG];
  bool qv[QG];
  float kM[QG], CM[QG], kQ[QG], CQ[QG];
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    const int i = qtile * p.q_per_cta + warp * QG + q;
    qv[q] = i < p.nq;
    qi[q] = min(i, p.nq - 1);
    const int vunit = (b * p.nq + qi[q]) * g.Hkv + h;
    const uint4* fr = reinterpret_cast<const uint4*>(p.ws.frag + (int64_t)vunit * (KS * 128));
    uint4* dst = s_frag4 + (size_t)(warp * QG + q) * (KS * 32);
    for (int k = lane; k < KS * 32; k += 32) dst[k] = fr[k];
    const float* qc = p.ws.qconst + ((int64_t)vunit * MG + tig) * 4;
    kM[q] = qc[0];
    CM[q] = qc[1];
    kQ[q] = qc[2];
    CQ[q] = qc[3];
  }
  __syncthreads();
  const uint4* bfr[QG];
#pragma unroll
  for (int q = 0; q < QG; ++q) bfr[q] = s_frag4 + (size_t)(warp * QG + q) * (KS * 32) + lane;

  const uint32_t maskA = 0x01010101u << tig, maskB = 0x10101010u << tig;
  // P V operands as in the decode: row gid (gid + 8) of m-tile mt is channel
  // 32 (mt >> 1) + 4 gid + 2 (mt & 1) (+1); a token-pair word shifted right by
  // 8 (gid & 1) and masked with 0x00030003 << 2k is code * 2^(2k - 24) of both
  // tokens.
  const uint32_t vshift = 8u * (uint32_t)(gid & 1);
  const int vc_lane = 16 * (gid >> 1);
  const float oddf = (gid & 1) ? 1.f : 0.f;
  const int hP = gid >> 1;

  float m_run[QG], l_run[QG];
  float acc[QG][8][4];
  float mnacc[QG][4];
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    m_run[q] = -INFINITY;
    l_run[q] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[q][i][c] = 0.f;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) mnacc[q][gi] = 0.f;
  }
  constexpr float kLazy = 4.f;     // the running max is raised only by more than this (log2)

  for (int j = 0; j < nb; ++j) {
    const int st = j % PNST;
    const uint32_t phase = (uint32_t)((j / PNST) & 1);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], phase));
    if (!ok && lane == 0) {
      atomicExch(p.err, 1);
      s_abort = 1;
    }
    if (ok) {
      const unsigned char* blk = stage + (size_t)st * bb;
      const int64_t tok0 = (blk0 + j) * kBlockTokens;
      const int nt_valid = (int)min((int64_t)kBlockTokens, p.n_comp - tok0);
      const float* rho = reinterpret_cast<const float*>(blk + g.o_rho);
      const float* rn = reinterpret_cast<const float*>(blk + g.o_rnorm);
      const float4* vm4 = reinterpret_cast<const float4*>(blk + g.o_vmin);
      const float4* vs4 = reinterpret_cast<const float4*>(blk + g.o_vscale);
      // two 16-token m-tiles per pass: every query-slice fragment loaded from shared
      // memory serves both, and the 8 MMAs of a k-step are independent
      for (int r2 = 0; r2 < kBlockTokens / 32; ++r2) {
        if (32 * r2 >= nt_valid) break;         // the rest of the block is past the end
        // rows of this lane: m-tile u (0, 1), row e (0: gid, 1: gid + 8)
        int tr[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e) tr[u][e] = 32 * r2 + 16 * u + gid + 8 * e;

        // ---------------- logits for the QG query tokens (head tig)
        float vM[2][QG][2] = {}, vQ[2][QG][2];
        if constexpr (KSM > 0) {
          int a[2][QG][2][4] = {};
#pragma unroll 1
          for (int c = 0; c < KSM; c += 4) {
            uint32_t w[2][2][4];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                lds_words<4>(blk + g.o_idx + tr[u][e] * (KSM * 4) + 4 * c, w[u][e]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              uint4 bq[QG];
#pragma unroll
              for (int q = 0; q < QG; ++q) bq[q] = bfr[q][(c + kk) * 32];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const uint32_t a0 = w[u][0][kk] & maskA, a1 = w[u][1][kk] & maskA;
                const uint32_t a2 = w[u][0][kk] & maskB, a3 = w[u][1][kk] & maskB;
#pragma unroll
                for (int q = 0; q < QG; ++q) {
                  imma16832(a[u][q][0], a0, a1, a2, a3, bq[q].x, bq[q].y);
                  imma16832(a[u][q][1], a0, a1, a2, a3, bq[q].z, bq[q].w);
                }
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < QG; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                vM[u][q][e] = slices_to_float(a[u][q][0][2 * e], a[u][q][0][2 * e + 1],
                                              a[u][q][1][2 * e], a[u][q][1][2 * e + 1]);
        }
        {
          constexpr int CQ4 = KSQ % 4 == 0 ? 4 : 2;
          int a[2][QG][2][4] = {};
#pragma unroll 1
          for (int c = 0; c < KSQ; c += CQ4) {
            uint32_t w[2][2][CQ4];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                lds_words<CQ4>(blk + g.o_sign + tr[u][e] * (KSQ * 4) + 4 * c, w[u][e]);
#pragma unroll
            for (int kk = 0; kk < CQ4; ++kk) {
              uint4 bq[QG];
#pragma unroll
              for (int q = 0; q < QG; ++q) bq[q] = bfr[q][(KSM + c + kk) * 32];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const uint32_t a0 = w[u][0][kk] & maskA, a1 = w[u][1][kk] & maskA;
                const uint32_t a2 = w[u][0][kk] & maskB, a3 = w[u][1][kk] & maskB;
#pragma unroll
                for (int q = 0; q < QG; ++q) {
                  imma16832(a[u][q][0], a0, a1, a2, a3, bq[q].x, bq[q].y);
                  imma16832(a[u][q][1], a0, a1, a2, a3, bq[q].z, bq[q].w);
                }
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < QG; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                vQ[u][q][e] = slices_to_float(a[u][q][0][2 * e], a[u][q][0][2 * e + 1],
                                              a[u][q][1][2 * e], a[u][q][1][2 * e + 1]);
        }

        // ---------------- softmax of the four rows (lazy running max per query token)
        float pr[2][QG][2];
#pragma unroll
        for (int q = 0; q < QG; ++q) {
          float l[2][2];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int t = tr[u][e];
              float v;
              if constexpr (B1 > 0)
                v = rho[t] * fmaf(kM[q], vM[u][q][e], CM[q]) + rn[t] * fmaf(kQ[q], vQ[u][q][e], CQ[q]);
              else
                v = rho[t] * fmaf(kQ[q], vQ[u][q][e], CQ[q]);
              l[u][e] = t >= nt_valid ? -INFINITY : v;
            }
          const float lmax = fmaxf(fmaxf(l[0][0], l[0][1]), fmaxf(l[1][0], l[1][1]));
          if (__any_sync(0xffffffffu, lmax > m_run[q] + kLazy)) {
            float mx = lmax;
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[q], mx);
            const float alpha = (m_run[q] == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f)
                                                        : exp2f(m_run[q] - m_new);
            m_run[q] = m_new;
            l_run[q] *= alpha;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[q][i][c] *= alpha;
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) mnacc[q][gi] *= alpha;
          }
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              pr[u][q][e] = m_run[q] == -INFINITY ? 0.f : exp2f(l[u][e] - m_run[q]);
          l_run[q] += (pr[0][q][0] + pr[0][q][1]) + (pr[1][q][0] + pr[1][q][1]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float4 mv = vm4[tr[u][e]];
#pragma unroll
            for (int q = 0; q < QG; ++q) {
              mnacc[q][0] = fmaf(pr[u][q][e], mv.x, mnacc[q][0]);
              mnacc[q][1] = fmaf(pr[u][q][e], mv.y, mnacc[q][1]);
              mnacc[q][2] = fmaf(pr[u][q][e], mv.z, mnacc[q][2]);
              mnacc[q][3] = fmaf(pr[u][q][e], mv.w, mnacc[q][3]);
            }
          }

        // ---------------- P V, one m-tile at a time: tokens TA = 16 (2 r2 + u) + 2 tig,
        // TA + 1, TC = TA + 8, TC + 1 are the MMA k indices of this lane
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int TA = 32 * r2 + 16 * u + 2 * tig, TC = TA + 8;
          const float4 sA = vs4[TA], sB = vs4[TA + 1], sC = vs4[TC], sD = vs4[TC + 1];
          const unsigned char* vc = blk + g.o_vcode + vc_lane;
          const uint4 wAB = *reinterpret_cast<const uint4*>(vc + (TA >> 1) * kPairBytes);
          const uint4 wCD = *reinterpret_cast<const uint4*>(vc + (TC >> 1) * kPairBytes);
          const uint32_t ab[4] = {wAB.x >> vshift, wAB.y >> vshift, wAB.z >> vshift, wAB.w >> vshift};
          const uint32_t cd[4] = {wCD.x >> vshift, wCD.y >> vshift, wCD.z >> vshift, wCD.w >> vshift};
          const float sa[4] = {sA.x, sA.y, sA.z, sA.w}, sb[4] = {sB.x, sB.y, sB.z, sB.w};
          const float sc[4] = {sC.x, sC.y, sC.z, sC.w}, sd[4] = {sD.x, sD.y, sD.z, sD.w};
          const float2 nodd = make_float2(-oddf, -oddf);
          uint32_t bpv[QG][4][2];
#pragma unroll
          for (int q = 0; q < QG; ++q) {
            const float pA = __shfl_sync(0xffffffffu, pr[u][q][0], 8 * tig + hP);
            const float pB = __shfl_sync(0xffffffffu, pr[u][q][0], 8 * tig + 4 + hP);
            const float pC = __shfl_sync(0xffffffffu, pr[u][q][1], 8 * tig + hP);
            const float pD = __shfl_sync(0xffffffffu, pr[u][q][1], 8 * tig + 4 + hP);
            const float2 pAB = make_float2(pA, pB), pCD = make_float2(pC, pD);
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              // column gid even carries fp16(p s), odd carries fp16(p s - fp16(p s))
              const float2 x0 = mul2(pAB, make_float2(sa[gi], sb[gi]));
              const float2 x1 = mul2(pCD, make_float2(sc[gi], sd[gi]));
              const float2 f0 = __half22float2(__floats2half2_rn(x0.x, x0.y));
              const float2 f1 = __half22float2(__floats2half2_rn(x1.x, x1.y));
              const float2 y0 = fma2(nodd, f0, x0), y1 = fma2(nodd, f1, x1);
              __half2 h0 = __floats2half2_rn(y0.x, y0.y);
              __half2 h1 = __floats2half2_rn(y1.x, y1.y);
              bpv[q][gi][0] = *reinterpret_cast<uint32_t*>(&h0);
              bpv[q][gi][1] = *reinterpret_cast<uint32_t*>(&h1);
            }
          }
          // one masked code operand serves both query tokens
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int gi = mt >> 1;
            const uint32_t m0 = 0x00030003u << (4 * (mt & 1)), m1 = m0 << 2;
            const uint32_t x0 = ab[gi] & m0, x1 = ab[gi] & m1, x2 = cd[gi] & m0, x3 = cd[gi] & m1;
#pragma unroll
            for (int q = 0; q < QG; ++q)
              hmma16816(acc[q][mt], x0, x1, x2, x3, bpv[q][gi][0], bpv[q][gi][1]);
          }
        }
      }
    }  // ok
    // release the stage; the last of the nw warps to finish it refills it
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int done = atomicAdd(&s_cnt[st], 1);
      if (done == nw - 1) {
        __threadfence_block();
        s_cnt[st] = 0;
        if (j + PNST < nb && !s_abort) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_expect_tx(&full[st], (uint32_t)bb);
          cache_bulk_load(stage + (size_t)st * bb, region + (blk0 + j + PNST) * bb, (uint32_t)bb,
                    &full[st], p.base, g.total_bytes, 303);
          s_iss[st] += 1;
        }
      }
    }
    if (*((volatile int*)&s_abort)) break;
  }
  __syncthreads();
  if (s_abort) {
    // a wait gave up: wait (bounded) for the last copy issued into every stage
    if (tid == 0)
      for (int s = 0; s < PNST; ++s)
        if (s_iss[s] > 0) (void)mbar_wait(&full[s], (uint32_t)((s_iss[s] - 1) & 1));
    return;
  }

  // ---------------- this warp's partials: (m, l) per head, o per head and channel
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    float l = l_run[q];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    float mn[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      float v = mnacc[q][gi];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      mn[gi] = v;
    }
    if (!qv[q]) continue;
    const int64_t slot = ((int64_t)(b * p.nq + qi[q]) * p.Hq + h * MG + tig) * p.nslots + split;
    float* po = p.ws.part_o + slot * MD;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int ch = 32 * (mt >> 1) + 4 * gid + 2 * (mt & 1);
      const float inv = __int_as_float((127 + 24 - 4 * (mt & 1)) << 23);   // 2^(24 - 2k)
      const float o0 = (acc[q][mt][0] + acc[q][mt][1]) * inv + mn[mt >> 1];
      const float o1 = (acc[q][mt][2] + acc[q][mt][3]) * (0.25f * inv) + mn[mt >> 1];
      *reinterpret_cast<float2*>(po + ch) = make_float2(o0, o1);
    }
    if (gid == 0) {
      p.ws.part_ml[slot * 2 + 0] = m_run[q];
      p.ws.part_ml[slot * 2 + 1] = l;
    }
  }
}

// ---------------------------------------------------------------- exact segment
struct EParams {
  Geom g;
  const uint8_t* base;
  int64_t n_total;        // tokens in the cache
  int n_ring, nq, Hq, G;
  const void* Knew;       // [B, Hkv, nq, d] in the cache dtype
  const void* Vnew;
  float scale_log2;
  int nslots, slot;
  DecodeWs ws;
};

constexpr int ET = 128;            // threads of the exact kernel
constexpr int ECH = 32;            // exact tokens per step

// One CTA per (query token i, batch, KV head): the G heads of query i over the ring
// tokens (oldest first) and chunk tokens 0..i, online softmax in chunks of ECH.
__global__ void __launch_bounds__(ET) k_prefill_exact(EParams p) {
  const Geom& g = p.g;
  const int d = g.d, G = p.G;
  const int i = blockIdx.x, unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ float s_q[kMaxG * 256];
  __shared__ float s_l[kMaxG][ECH], s_p[kMaxG][ECH];
  __shared__ float s_m[kMaxG], s_ls[kMaxG], s_al[kMaxG];
  const int64_t bq0 = (int64_t)(b * p.nq + i) * p.Hq + h * G;
  for (int k = tid; k < G * d; k += ET) s_q[k] = p.ws.qf[bq0 * d + k];
  if (tid < kMaxG) {
    s_m[tid] = -INFINITY;
    s_ls[tid] = 0.f;
    s_al[tid] = 1.f;
  }
  __syncthreads();
  const int64_t first = p.n_total - p.n_ring;      // absolute index of the oldest ring token
  const int n_ex = p.n_ring + i + 1;
  // element e of exact token t's key or value row
  auto row_ptr = [&](int t, bool key, int64_t& e) -> const void* {
    if (t < p.n_ring) {
      const int64_t slot = (first + t) % g.W;
      e = ((int64_t)unit * g.W + slot) * d;
      return p.base + (key ? g.ring_k_off : g.ring_v_off);
    }
    e = ((int64_t)unit * p.nq + (t - p.n_ring)) * d;
    return key ? p.Knew : p.Vnew;
  };
  float acc[kMaxG][2];
#pragma unroll
  for (int k = 0; k < kMaxG; ++k) acc[k][0] = acc[k][1] = 0.f;

  for (int c0 = 0; c0 < n_ex; c0 += ECH) {
    const int rows = min(ECH, n_ex - c0);
    for (int tt = warp; tt < ECH; tt += ET / 32) {
      if (tt < rows) {
        int64_t e;
        const void* kp = row_ptr(c0 + tt, true, e);
        float kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) kv[u] = (lane + 32 * u < d) ? load_f(kp, e + lane + 32 * u, g.dtype) : 0.f;
        for (int hh = 0; hh < G; ++hh) {
          float dot = 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (lane + 32 * u < d) dot = fmaf(s_q[hh * d + lane + 32 * u], kv[u], dot);
          dot = warp_sum(dot);
          if (lane == 0) s_l[hh][tt] = dot * p.scale_log2;
        }
      } else if (lane < G) {
        s_l[lane][tt] = -INFINITY;
      }
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += ET / 32) {
      const float v = s_l[hh][lane];
      const float mx = warp_max(v);
      const float m_old = s_m[hh], m_new = fmaxf(m_old, mx);
      const float alpha = exp2f(m_old - m_new);          // m_new is finite: rows >= 1
      const float pv = exp2f(v - m_new);
      const float sum = warp_sum(pv);
      s_p[hh][lane] = pv;
      if (lane == 0) {
        s_ls[hh] = s_ls[hh] * alpha + sum;
        s_m[hh] = m_new;
        s_al[hh] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int ch = tid + ET * u;
      if (ch >= d) break;
#pragma unroll
      for (int k = 0; k < kMaxG; ++k)
        if (k < G) acc[k][u] *= s_al[k];
      for (int tt = 0; tt < rows; ++tt) {
        int64_t e;
        const void* vp = row_ptr(c0 + tt, false, e);
        const float v = load_f(vp, e + ch, g.dtype);
#pragma unroll
        for (int k = 0; k < kMaxG; ++k)
          if (k < G) acc[k][u] = fmaf(s_p[k][tt], v, acc[k][u]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int ch = tid + ET * u;
    if (ch >= d) break;
#pragma unroll
    for (int k = 0; k < kMaxG; ++k)
      if (k < G) p.ws.part_o[((bq0 + k) * p.nslots + p.slot) * d + ch] = acc[k][u];
  }
  if (tid < G) {
    p.ws.part_ml[((bq0 + tid) * p.nslots + p.slot) * 2 + 0] = s_m[tid];
    p.ws.part_ml[((bq0 + tid) * p.nslots + p.slot) * 2 + 1] = s_ls[tid];
  }
}

template <int B1, int KSQ>
cudaError_t launch_prefill_t(const PParams& p, int nw, cudaStream_t s) {
  constexpr int KS = (B1 > 0 ? (1 << (B1 - 1)) * MD / 32 : 0) + KSQ;
  const size_t smem = (size_t)PNST * p.g.block_bytes + (size_t)nw * QG * KS * 128 * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(k_prefill_partial_mma<B1, KSQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int qtiles = (p.nq + p.q_per_cta - 1) / p.q_per_cta;
  dim3 grid((unsigned)qtiles, (unsigned)p.splits, (unsigned)(p.g.B * p.g.Hkv));
  return launch_pdl(k_prefill_partial_mma<B1, KSQ>, grid, dim3(32 * nw), smem, s, p);
}

}  // namespace

bool prefill_mma_supported(const Geom& g, int G) {
  return g.d == MD && G == MG && g.vbits == 2 && g.group == 32 && g.b1 <= 2 &&
         (g.m == 64 || g.m == 128 || g.m == 192 || g.m == 256 || g.m == 384 || g.m == 512);
}

// Warps of the tensor-core partial: QG query tokens each, at most PNW, and no more
// than the shared memory holds (the staged blocks plus every warp's query slices).
int prefill_mma_warps(const Geom& g, int nq) {
  const int F = g.b1 > 0 ? 1 << (g.b1 - 1) : 0;
  const int KS = F * MD / 32 + g.m / 32;
  const size_t per_warp = (size_t)QG * KS * 128 * sizeof(uint32_t);
  const size_t avail = (size_t)226 * 1024 - (size_t)PNST * g.block_bytes;
  const int fit = (int)(avail / per_warp);
  return max(1, min(min(PNW, fit), (nq + QG - 1) / QG));
}

int prefill_auto_splits(const Geom& g, int G, int64_t n_comp, int nq, bool mma) {
  const int64_t nblk = (n_comp + kBlockTokens - 1) / kBlockTokens;
  if (nblk <= 1) return 1;
  const int units = g.B * g.Hkv;
  if (mma && prefill_tc_supported(g, G, nq)) return prefill_tc_splits(g, n_comp, nq);
  if (!mma) {
    // the CUDA-core partial runs per virtual (query token) batch: one wave or so
    int64_t s = (148 * 4 + (int64_t)units * nq - 1) / ((int64_t)units * nq);
    return (int)max((int64_t)1, min(nblk, s));
  }
  const int nw = prefill_mma_warps(g, nq);
  const int qpc = QG * nw;
  const int64_t base = (int64_t)units * ((nq + qpc - 1) / qpc);
  // resident CTAs per SM: registers and shared memory (staged blocks + query slices)
  const int F = g.b1 > 0 ? 1 << (g.b1 - 1) : 0;
  const int KS = F * MD / 32 + g.m / 32;
  const size_t smem = (size_t)PNST * g.block_bytes + (size_t)nw * QG * KS * 128 * sizeof(uint32_t);
  const int by_regs = 65536 / (nw * 32 * kPrefillRegs);
  const int by_smem = (int)((size_t)(227 * 1024) / (smem + 1024));
  const int slots = 148 * max(1, min(by_regs, by_smem));
  // the split count whose grid fills its last wave best, at least 4 blocks a split
  int best = 1;
  double best_score = -1.0;
  for (int s = 1; s <= 64 && s <= nblk; ++s) {
    if (s > 1 && nblk / s < 4) break;
    const int64_t ctas = base * s;
    const int64_t waves = (ctas + slots - 1) / slots;
    const double score = (double)ctas / (double)(waves * slots) - 0.002 * s;
    if (score > best_score) {
      best_score = score;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_prefill_partial_mma(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                       int nq, int splits, int nslots, const DecodeWs& ws,
                                       cudaStream_t s) {
  PParams p{};
  p.g = g;
  p.base = base;
  p.n_comp = n_total > g.W ? n_total - g.W : 0;
  p.nq = nq;
  p.Hq = Hq;
  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  p.splits = splits;
  p.nslots = nslots;
  p.bps = (int)((nblk + splits - 1) / splits);
  const int nw = prefill_mma_warps(g, nq);
  p.q_per_cta = QG * nw;
  p.ws = ws;
  p.err = ws.err;
  const int ksq = g.m / 32;
  switch (g.b1 * 32 + ksq) {
    case 0 * 32 + 2: return launch_prefill_t<0, 2>(p, nw, s);
    case 0 * 32 + 4: return launch_prefill_t<0, 4>(p, nw, s);
    case 0 * 32 + 6: return launch_prefill_t<0, 6>(p, nw, s);
    case 0 * 32 + 8: return launch_prefill_t<0, 8>(p, nw, s);
    case 0 * 32 + 12: return launch_prefill_t<0, 12>(p, nw, s);
    case 0 * 32 + 16: return launch_prefill_t<0, 16>(p, nw, s);
    case 1 * 32 + 2: return launch_prefill_t<1, 2>(p, nw, s);
    case 1 * 32 + 4: return launch_prefill_t<1, 4>(p, nw, s);
    case 1 * 32 + 6: return launch_prefill_t<1, 6>(p, nw, s);
    case 1 * 32 + 8: return launch_prefill_t<1, 8>(p, nw, s);
    case 1 * 32 + 12: return launch_prefill_t<1, 12>(p, nw, s);
    case 1 * 32 + 16: return launch_prefill_t<1, 16>(p, nw, s);
    case 2 * 32 + 2: return launch_prefill_t<2, 2>(p, nw, s);
    case 2 * 32 + 4: return launch_prefill_t<2, 4>(p, nw, s);
    case 2 * 32 + 6: return launch_prefill_t<2, 6>(p, nw, s);
    case 2 * 32 + 8: return launch_prefill_t<2, 8>(p, nw, s);
    case 2 * 32 + 12: return launch_prefill_t<2, 12>(p, nw, s);
    case 2 * 32 + 16: return launch_prefill_t<2, 16>(p, nw, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_prefill_exact(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                 int nq, const void* K, const void* V, float scale, int nslots,
                                 int slot, const DecodeWs& ws, cudaStream_t s) {
  EParams p{};
  p.g = g;
  p.base = base;
  p.n_total = n_total;
  p.n_ring = (int)(n_total < g.W ? n_total : g.W);
  p.nq = nq;
  p.Hq = Hq;
  p.G = Hq / g.Hkv;
  p.Knew = K;
  p.Vnew = V;
  p.scale_log2 = scale * kLog2e;
  p.nslots = nslots;
  p.slot = slot;
  p.ws = ws;
  dim3 grid((unsigned)nq, (unsigned)(g.B * g.Hkv));
  k_prefill_exact<<<grid, ET, 0, s>>>(p);
  return cudaGetLastError();
}

TQ_BOUNDS_READER(bounds_flag_prefill)

}  // namespace tq
