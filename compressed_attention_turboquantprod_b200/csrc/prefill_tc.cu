// Multi-token (chunked prefill) history partials with the scores on the
// fifth-generation tensor cores ([TQ] 四-六 estimator over the packed cache).
//
// A chunk of n new tokens is scored against the compressed history as n decode
// queries (virtual batch b n + i, prepared by the decode's query preparation).
// In the decode one stored key operand serves a single query, so expanding the
// bits into MMA operands is most of the work; here one 128-token tile of the
// history serves NQ = 16 query tokens, so the expansion is paid once per tile and
// the contraction goes to tcgen05:
//
//   D[128 tokens x 16 NQ columns per kind] = A[128 tokens x K] . B[K x 16 NQ]
//     A = the tokens' stored feature bits as unsigned bytes in shared memory:
//         K byte 32 k + 4 t + b of a token = bit t of byte b of its stored word k
//         (feature 32 k + 8 b + t), value 2^t (one AND per four features);
//     B = per (query token, head) the 24-bit fixed-point query weights of those
//         features times 2^(7 - t) as four signed int8 slices (column
//         16 q + 4 h + slice), built once per CTA from the prepared Pi q and
//         sqrt(pi/2)/m S q exactly as the decode's preparation quantises them;
//     the MSE features accumulate into columns 0..255 and the QJL features into
//     256..511 (different per-token factors rho and ||r||), exact int32 in
//     tensor memory, kind::i8, M = 128, N = 256, K = 32 per instruction.
//
// Each token's thread pair expands the bits, one thread issues the MMAs, then
// every thread reads its token row back (tcgen05.ld), joins the slices into the
// logits of 16 query tokens x 4 heads and leaves them in shared memory; the
// online softmax and P V then run per query token on warp-level MMA exactly as in
// the decode (value codes as f16 subnormals from the token-pair records, B =
// p * s split into f16 hi + lo), two query tokens per warp.
//
// Specialisation: head dim 128, G = 4, 2-bit values in groups of 32, b1 in
// {0, 1, 2}, 32 (b1 planes x 4 + m / 32) <= 384 K bytes (the A and B operands
// fit in shared memory beside the staged tiles).  Other shapes use
// k_prefill_partial_mma.
#include <cfloat>

#include "mma_common.cuh"
#include "tc_common.cuh"

namespace tq {
namespace {
using namespace mmadec;

constexpr int TD = 128;                    // head dim
constexpr int TNQ = 16;                    // query tokens per CTA
constexpr int TTH = 256;                   // threads (8 warps)
constexpr int TTOK = 128;                  // history tokens per tile (MMA M)
constexpr int TNCOL = TNQ * 16;            // accumulator columns per kind (q, head, slice)
constexpr int TNST = 3;                    // staged tiles
constexpr int kTPairBytes = 2 * TD * 2 / 8;
constexpr int TLS = TNQ * 4 + 4;           // row stride (floats) of the tile's logits: rows 4 banks apart

struct TParams {
  Geom g;
  const uint8_t* base;
  int64_t n_comp;         // compressed tokens
  int nq, Hq;             // chunk length, query heads
  int splits, nslots, bps;   // bps: blocks per split (even)
  const float* cent;      // codebook (b1 > 0)
  DecodeWs ws;            // carved for the virtual batch B * nq
  int* err;
};

__host__ __device__ constexpr int tc_ks(int b1, int ksq) { return (b1 > 0 ? (1 << (b1 - 1)) * 4 : 0) + ksq; }

// Dynamic shared memory: B operand (256 rows), A operand (128 rows), TNST staged
// tiles of two cache blocks, the logits of a tile (128 tokens x 64 (query, head)).
__host__ __device__ inline size_t tc_prefill_smem(int ks, int64_t block_bytes) {
  return (size_t)TNCOL * 32 * ks + (size_t)TTOK * 32 * ks + (size_t)TNST * 2 * block_bytes +
         sizeof(float) * TTOK * TLS;
}

// Byte offset of 16-byte chunk kc of row r in a canonical K-major operand of kb
// bytes per row (8-row x 16-byte core matrices, row groups 8 kb bytes apart).
__device__ __forceinline__ int op_off(int r, int kc, int kb) {
  return ((r >> 3) * (kb >> 4) + kc) * 128 + (r & 7) * 16;
}

__device__ __forceinline__ uint64_t op_desc(uint32_t saddr, int kb) {
  return tc::smem_desc_sbo(saddr, (uint32_t)(8 * kb));
}

template <int B1, int KSQ>
__global__ void __launch_bounds__(TTH, 1) k_prefill_partial_tc(TParams p) {
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;
  constexpr int KSM = F * TD / 32;           // MSE k-steps (stored words)
  constexpr int KS = KSM + KSQ;
  constexpr int KB = 32 * KS;                // K bytes per row
  constexpr uint32_t kCols = B1 > 0 ? 2 * TNCOL : TNCOL;
  constexpr uint32_t kColQ = B1 > 0 ? TNCOL : 0;   // first QJL accumulator column
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_full[TNST];
  __shared__ __align__(8) uint64_t s_mma;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort, s_iss[TNST];
  __shared__ float s_w[4];
  __shared__ float s_mx[TNQ * MG][2];        // per (query, head): largest |MSE|, |QJL| weight
  __shared__ float4 s_qc[TNQ * MG];          // per (query, head): kM, CM, kQ, CQ

  const Geom& g = p.g;
  const int qgrp = blockIdx.x, split = blockIdx.y, unit = blockIdx.z;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bb = (int)g.block_bytes;
  unsigned char* SB = smem_raw;                                   // [256 rows][KB]
  unsigned char* SA = SB + TNCOL * KB;                            // [128 rows][KB]
  unsigned char* ST = SA + TTOK * KB;                             // [TNST][2 blocks]
  float* SL = reinterpret_cast<float*>(ST + (size_t)TNST * 2 * bb);   // [128 tokens][16 q][4 h]

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
  const int ntiles = (nb + 1) / 2;
  const uint8_t* region = p.base + (int64_t)unit * g.region_bytes;

  if (tid == 0) {
    for (int s = 0; s < TNST; ++s) mbar_init(&s_full[s], 1);
    mbar_init(&s_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(&s_tmem), kCols);
    tc::tmem_relinquish();
  }
  // launched programmatically after the query preparation
  pdl_wait();
  auto load_tile = [&](int j, int s) {       // blocks 2j, 2j+1 of the split: adjacent in memory
    const int nbt = min(2, nb - 2 * j);
    const uint32_t bytes = (uint32_t)(nbt * bb);
    mbar_expect_tx(&s_full[s], bytes);
    cache_bulk_load(ST + (size_t)s * 2 * bb, region + (blk0 + 2 * j) * bb, bytes, &s_full[s], p.base,
                    g.total_bytes, 321);
  };
  if (tid == 0) {
    for (int s = 0; s < TNST; ++s) {
      s_iss[s] = 0;
      if (s < ntiles) {
        load_tile(s, s);
        s_iss[s] = 1;
      }
    }
  }
  // ---- the query side, once per CTA.  Query token i of this group (a token past the
  // chunk end repeats the last one and is not written) is virtual batch b nq + i.
  if (tid < 4) {
    // Walsh weights of the codebook, as the decode's preparation computes them
    const int L = B1 > 0 ? 1 << B1 : 0;
    const int subset = tid < 3 ? 1 << tid : 7;
    double acc = 0.0;
    for (int idx = 0; idx < L; ++idx)
      acc += (double)p.cent[idx] * ((__popc(idx & subset) & 1) ? -1.0 : 1.0);
    s_w[tid] = L ? (float)(acc / L) : 0.f;
  }
  __syncthreads();
  auto qrow = [&](int q) {                   // virtual query row of (query token q, head 0)
    const int i = min(qgrp * TNQ + q, p.nq - 1);
    return (int64_t)(b * p.nq + i) * p.Hq + h * MG;
  };
  {
    float wk = 0.f;
#pragma unroll
    for (int k = 0; k < F; ++k) wk = fmaxf(wk, fabsf(2.f * s_w[k]));
    // per (query, head): the largest weight magnitude of each kind (one warp each)
    for (int pr = warp; pr < TNQ * MG; pr += TTH / 32) {
      const int q = pr >> 2, hh = pr & 3;
      const int64_t row = qrow(q) + hh;
      float mM = 0.f, mQ = 0.f;
      if (F)
        for (int j = lane; j < TD; j += 32) mM = fmaxf(mM, wk * fabsf(p.ws.qr[row * TD + j]));
      for (int i = lane; i < g.m; i += 32) mQ = fmaxf(mQ, fabsf(2.f * p.ws.qs[row * g.m + i]));
      mM = warp_max(mM);
      mQ = warp_max(mQ);
      if (lane == 0) {
        s_mx[pr][0] = mM;
        s_mx[pr][1] = mQ;
        const int i = min(qgrp * TNQ + q, p.nq - 1);
        const float* c = p.ws.qconst + ((int64_t)((b * p.nq + i) * g.Hkv + h) * MG + hh) * 4;
        s_qc[pr] = make_float4(c[0], c[1], c[2], c[3]);
      }
    }
  }
  __syncthreads();
  {
    // B: rows 16 q + 4 hh + slice, 16-byte chunks kc of stored word ks = kc / 2;
    // byte 4 t' + b of the chunk is feature 32 ks + 8 b + t (t = 4 (kc & 1) + t'),
    // weight rint(w kFix / max) 2^(7 - t) split into four int8 slices
    const float kFix = 16646144.f;
    for (int it = tid; it < TNQ * MG * (KB / 16); it += TTH) {
      const int kc = it % (KB / 16), pr = it / (KB / 16);
      const int q = pr >> 2, hh = pr & 3;
      const int ks = kc >> 1;
      const bool mse = ks < KSM;
      const float mx = s_mx[pr][mse ? 0 : 1];
      const float inv_delta = mx > 0.f ? kFix / mx : 1.f;
      const int64_t row = qrow(q) + hh;
      const float wsc = mse ? -2.f * s_w[ks / (TD / 32)] : 2.f;
      const float* src = mse ? p.ws.qr + row * TD + 32 * (ks % (TD / 32))
                             : p.ws.qs + row * g.m + 32 * (ks - KSM);
      uint32_t sl[4][4];                       // [slice][word of the chunk]
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = 4 * (kc & 1) + tt;
#pragma unroll
        for (int s = 0; s < 4; ++s) sl[s][tt] = 0u;
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
          const float w = wsc * src[8 * bq + t];
          const int wint = __float2int_rn(w * inv_delta) * (1 << (7 - t));   // |wint| < 2^31
          const int s0 = ((wint + 128) & 255) - 128;
          const int t1 = (wint - s0) >> 8;
          const int s1 = ((t1 + 128) & 255) - 128;
          const int t2 = (t1 - s1) >> 8;
          const int s2 = ((t2 + 128) & 255) - 128;
          const int s3 = (t2 - s2) >> 8;
          sl[0][tt] |= (uint32_t)(s0 & 255) << (8 * bq);
          sl[1][tt] |= (uint32_t)(s1 & 255) << (8 * bq);
          sl[2][tt] |= (uint32_t)(s2 & 255) << (8 * bq);
          sl[3][tt] |= (uint32_t)(s3 & 255) << (8 * bq);
        }
      }
#pragma unroll
      for (int s = 0; s < 4; ++s)
        *reinterpret_cast<uint4*>(SB + op_off(16 * q + 4 * hh + s, kc, KB)) =
            make_uint4(sl[s][0], sl[s][1], sl[s][2], sl[s][3]);
    }
  }
  tc::fence_async_shared();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t sA = smem_u32(SA), sB = smem_u32(SB);

  // P V operands in the lane layout of the warp-level MMAs (as in the decode)
  const int gid = lane >> 2, tig = lane & 3;
  const uint32_t vshift = 8u * (uint32_t)(gid & 1);
  const int vc_lane = 16 * (gid >> 1);
  const float oddf = (gid & 1) ? 1.f : 0.f;
  const int hP = gid >> 1;
  constexpr int QW = 2;                      // query tokens per warp in the softmax and P V
  const int q0 = QW * warp;
  float m_run[QW], l_run[QW], acc[QW][8][4], mnacc[QW][4];
#pragma unroll
  for (int q = 0; q < QW; ++q) {
    m_run[q] = -INFINITY;
    l_run[q] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[q][i][c] = 0.f;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) mnacc[q][gi] = 0.f;
  }
  constexpr float kLazy = 4.f;               // the running max is raised only by more than this
  const int xt = tid >> 1, xh = tid & 1;     // expansion: token xt, half xh of its stored words
  const int lt = 32 * (warp & 3) + lane;     // logits: the token of this tensor-memory lane
  const int lqh = warp >> 2;                 // and the half of the query tokens
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  int mma_issued = 0;
  auto tile_nbt = [&](int j) { return min(2, nb - 2 * j); };       // staged blocks of tile j
  auto tile_ptr = [&](int j) { return ST + (size_t)(j % TNST) * 2 * bb; };
  // A of tile j from its staged bits (a second block that is not staged: zero),
  // then one thread issues the tile's products into tensor memory
  auto expand_and_issue = [&](int j) {
    if (!mbar_wait(&s_full[j % TNST], (uint32_t)((j / TNST) & 1))) {
      atomicExch(p.err, 1);
      s_abort = 1;
    }
    const int bi = xt >> 6, tb = xt & 63;
    const unsigned char* blk = tile_ptr(j) + bi * bb;
    const bool have = bi < tile_nbt(j);
#pragma unroll
    for (int k = 0; k < KS / 2; ++k) {
      const int ks = xh * (KS / 2) + k;
      uint32_t w = 0u;
      if (have)
        w = ks < KSM ? *reinterpret_cast<const uint32_t*>(blk + g.o_idx + tb * (KSM * 4) + 4 * ks)
                     : *reinterpret_cast<const uint32_t*>(blk + g.o_sign + tb * (KSQ * 4) + 4 * (ks - KSM));
      *reinterpret_cast<uint4*>(SA + op_off(xt, 2 * ks, KB)) =
          make_uint4(w & 0x01010101u, w & 0x02020202u, w & 0x04040404u, w & 0x08080808u);
      *reinterpret_cast<uint4*>(SA + op_off(xt, 2 * ks + 1, KB)) =
          make_uint4(w & 0x10101010u, w & 0x20202020u, w & 0x40404040u, w & 0x80808080u);
    }
    tc::fence_async_shared();
    tc::fence_before_sync();
    __syncthreads();
    if (*reinterpret_cast<volatile int*>(&s_abort)) return;
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t idesc = tc::idesc_i8_us(TTOK, TNCOL);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
        tc::mma_i8(tmem + (ks < KSM ? 0u : kColQ), op_desc(sA + 256u * ks, KB), op_desc(sB + 256u * ks, KB),
                   idesc, (ks == 0 || ks == KSM) ? 0u : 1u);
      tc::mma_commit(smem_u32(&s_mma));
    }
    ++mma_issued;
  };

  // Tile j's products run while the warps work through the softmax and P V of
  // tile j - 1: its A is written (and its products issued) as soon as the logits
  // of tile j - 1 have left tensor memory.
  if (ntiles > 0) expand_and_issue(0);
  for (int j = 0; j < ntiles; ++j) {
    if (*reinterpret_cast<volatile int*>(&s_abort)) break;
    const int st = j % TNST;
    const int nbt = tile_nbt(j);
    const int64_t tok0 = (blk0 + 2 * j) * kBlockTokens;
    const int nvalid = (int)min((int64_t)(kBlockTokens * nbt), p.n_comp - tok0);
    const unsigned char* tile = tile_ptr(j);
    if (!mbar_wait_sleep(&s_mma, (uint32_t)(j & 1))) {
      atomicExch(p.err, 1);
      s_abort = 1;
    }
    tc::fence_after_sync();
    // ---- logits of this thread's token for its 8 query tokens x 4 heads
    {
      const int bi = lt >> 6, tb = lt & 63;
      const unsigned char* blk = tile + bi * bb;
      const bool valid = lt < nvalid;
      const float rho = valid ? reinterpret_cast<const float*>(blk + g.o_rho)[tb] : 0.f;
      const float rn = valid && B1 > 0 ? reinterpret_cast<const float*>(blk + g.o_rnorm)[tb] : 0.f;
#pragma unroll 2
      for (int qq = 0; qq < TNQ / 2; ++qq) {
        const int q = (TNQ / 2) * lqh + qq;
        uint32_t vq[16], vm[16];
        tc::tmem_ld16(trow + kColQ + 16u * q, vq);
        if constexpr (B1 > 0) tc::tmem_ld16(trow + 16u * q, vm);
        tc::tmem_wait_ld();
        float l[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float4 c = s_qc[4 * q + hh];
          const float vQ = slices_to_float((int)vq[4 * hh], (int)vq[4 * hh + 1], (int)vq[4 * hh + 2],
                                           (int)vq[4 * hh + 3]);
          float v;
          if constexpr (B1 > 0) {
            const float vM = slices_to_float((int)vm[4 * hh], (int)vm[4 * hh + 1], (int)vm[4 * hh + 2],
                                             (int)vm[4 * hh + 3]);
            v = rho * fmaf(c.x, vM, c.y) + rn * fmaf(c.z, vQ, c.w);
          } else {
            v = rho * fmaf(c.z, vQ, c.w);
          }
          l[hh] = valid ? v : -INFINITY;
        }
        *reinterpret_cast<float4*>(SL + lt * TLS + 4 * q) = make_float4(l[0], l[1], l[2], l[3]);
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    // tensor memory and A are free: the next tile's products start now
    if (j + 1 < ntiles) expand_and_issue(j + 1);
    // ---- softmax and P V of this warp's two query tokens over the tile's tokens
    for (int bi = 0; bi < nbt; ++bi) {
      const unsigned char* blk = tile + bi * bb;
      const int bvalid = nvalid - kBlockTokens * bi;
      const float4* vm4 = reinterpret_cast<const float4*>(blk + g.o_vmin);
      const float4* vs4 = reinterpret_cast<const float4*>(blk + g.o_vscale);
      for (int r2 = 0; r2 < kBlockTokens / 32; ++r2) {
        if (32 * r2 >= bvalid) break;          // the rest of the block is past the end
        int tr[2][2];                          // rows of this lane: m-tile u, row e
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e) tr[u][e] = 32 * r2 + 16 * u + gid + 8 * e;
        float pr[2][QW][2];
#pragma unroll
        for (int q = 0; q < QW; ++q) {
          float l[2][2];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 2; ++e) l[u][e] = SL[(kBlockTokens * bi + tr[u][e]) * TLS + 4 * (q0 + q) + tig];
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
        // the value minima enter as sum_t p_t mn_{t,g} per head (tig) and group
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float4 mv = vm4[tr[u][e]];
#pragma unroll
            for (int q = 0; q < QW; ++q) {
              mnacc[q][0] = fmaf(pr[u][q][e], mv.x, mnacc[q][0]);
              mnacc[q][1] = fmaf(pr[u][q][e], mv.y, mnacc[q][1]);
              mnacc[q][2] = fmaf(pr[u][q][e], mv.z, mnacc[q][2]);
              mnacc[q][3] = fmaf(pr[u][q][e], mv.w, mnacc[q][3]);
            }
          }
        // P V, one 16-token m-tile at a time: tokens TA = 32 r2 + 16 u + 2 tig, TA + 1,
        // TC = TA + 8, TC + 1 are the MMA k indices of this lane
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int TA = 32 * r2 + 16 * u + 2 * tig, TC = TA + 8;
          const float4 sA4 = vs4[TA], sB4 = vs4[TA + 1], sC4 = vs4[TC], sD4 = vs4[TC + 1];
          const unsigned char* vc = blk + g.o_vcode + vc_lane;
          const uint4 wAB = *reinterpret_cast<const uint4*>(vc + (TA >> 1) * kTPairBytes);
          const uint4 wCD = *reinterpret_cast<const uint4*>(vc + (TC >> 1) * kTPairBytes);
          const uint32_t ab[4] = {wAB.x >> vshift, wAB.y >> vshift, wAB.z >> vshift, wAB.w >> vshift};
          const uint32_t cd[4] = {wCD.x >> vshift, wCD.y >> vshift, wCD.z >> vshift, wCD.w >> vshift};
          const float sa[4] = {sA4.x, sA4.y, sA4.z, sA4.w}, sb[4] = {sB4.x, sB4.y, sB4.z, sB4.w};
          const float sc[4] = {sC4.x, sC4.y, sC4.z, sC4.w}, sd[4] = {sD4.x, sD4.y, sD4.z, sD4.w};
          const float2 nodd = make_float2(-oddf, -oddf);
          uint32_t bpv[QW][4][2];
#pragma unroll
          for (int q = 0; q < QW; ++q) {
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
            for (int q = 0; q < QW; ++q) hmma16816(acc[q][mt], x0, x1, x2, x3, bpv[q][gi][0], bpv[q][gi][1]);
          }
        }
      }
    }
    // every read of the staged tile is done: refill its stage with tile j + TNST
    __syncthreads();
    if (tid == 0 && j + TNST < ntiles && !*reinterpret_cast<volatile int*>(&s_abort)) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      load_tile(j + TNST, st);
      s_iss[st] += 1;
    }
  }
  __syncthreads();
  if (s_abort) {
    // a wait gave up: let the products and copies in flight finish (bounded), free
    // the tensor memory and leave
    if (tid == 0) {
      if (mma_issued > 0) (void)mbar_wait(&s_mma, (uint32_t)((mma_issued - 1) & 1));
      for (int s = 0; s < TNST; ++s)
        if (s_iss[s] > 0) (void)mbar_wait(&s_full[s], (uint32_t)((s_iss[s] - 1) & 1));
    }
    __syncthreads();
    if (warp == 0) {
      tc::fence_after_sync();
      tc::tmem_dealloc(tmem, kCols);
    }
    return;
  }

  // ---------------- this warp's partials: (m, l) per head, o per head and channel
#pragma unroll
  for (int q = 0; q < QW; ++q) {
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
    const int i = qgrp * TNQ + q0 + q;
    if (i >= p.nq) continue;
    const int64_t slot = ((int64_t)(b * p.nq + i) * p.Hq + h * MG + tig) * p.nslots + split;
    float* po = p.ws.part_o + slot * TD;
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
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
}

template <int B1, int KSQ>
cudaError_t launch_tc_t(const TParams& p, cudaStream_t s) {
  constexpr int KS = tc_ks(B1, KSQ);
  const size_t smem = tc_prefill_smem(KS, p.g.block_bytes);
  cudaError_t e = cudaFuncSetAttribute(k_prefill_partial_tc<B1, KSQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.nq + TNQ - 1) / TNQ), (unsigned)p.splits, (unsigned)(p.g.B * p.g.Hkv));
  return launch_pdl(k_prefill_partial_tc<B1, KSQ>, grid, dim3(TTH), smem, s, p);
}

}  // namespace

// The tcgen05 history partial: the decode's tensor-core shapes whose operands fit
// (K bytes 32 (b1 planes x 4 + m / 32) <= 384), for chunks of at least 8 tokens
// (a query group is 16 tokens; below 8 most of its B operand would be padding).
bool prefill_tc_supported(const Geom& g, int G, int nq) {
  if (!(g.d == TD && G == MG && g.vbits == 2 && g.group == 32 && g.b1 <= 2)) return false;
  if (!(g.m == 64 || g.m == 128 || g.m == 192 || g.m == 256 || g.m == 384)) return false;
  const int ks = tc_ks(g.b1, g.m / 32);
  if (ks > 12 || tc_prefill_smem(ks, g.block_bytes) > (size_t)225 * 1024) return false;
  return nq >= 8;
}

// Splits of the tcgen05 partial: one CTA per SM, at least two 128-token tiles a
// split, the count whose grid fills its last wave best.
int prefill_tc_splits(const Geom& g, int64_t n_comp, int nq) {
  const int64_t nblk = (n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t ntiles = (nblk + 1) / 2;
  if (ntiles <= 2) return 1;
  const int64_t base = (int64_t)g.B * g.Hkv * ((nq + TNQ - 1) / TNQ);
  int best = 1;
  double best_score = -1.0;
  for (int s = 1; s <= 64 && s <= ntiles; ++s) {
    if (s > 1 && ntiles / s < 2) break;
    const int64_t ctas = base * s;
    const int64_t waves = (ctas + 147) / 148;
    const double score = (double)ctas / (double)(waves * 148) - 0.002 * s;
    if (score > best_score) {
      best_score = score;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_prefill_partial_tc(const Geom& g, const uint8_t* base, int64_t n_total, int Hq, int nq,
                                      int splits, int nslots, const float* cent, const DecodeWs& ws,
                                      cudaStream_t s) {
  TParams p{};
  p.g = g;
  p.base = base;
  p.n_comp = n_total > g.W ? n_total - g.W : 0;
  p.nq = nq;
  p.Hq = Hq;
  p.splits = splits;
  p.nslots = nslots;
  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t ntiles = (nblk + 1) / 2;
  p.bps = (int)(2 * ((ntiles + splits - 1) / splits));     // whole tiles per split
  p.cent = cent;
  p.ws = ws;
  p.err = ws.err;
  switch (g.b1 * 32 + g.m / 32) {
    case 0 * 32 + 2: return launch_tc_t<0, 2>(p, s);
    case 0 * 32 + 4: return launch_tc_t<0, 4>(p, s);
    case 0 * 32 + 6: return launch_tc_t<0, 6>(p, s);
    case 0 * 32 + 8: return launch_tc_t<0, 8>(p, s);
    case 0 * 32 + 12: return launch_tc_t<0, 12>(p, s);
    case 1 * 32 + 2: return launch_tc_t<1, 2>(p, s);
    case 1 * 32 + 4: return launch_tc_t<1, 4>(p, s);
    case 1 * 32 + 6: return launch_tc_t<1, 6>(p, s);
    case 1 * 32 + 8: return launch_tc_t<1, 8>(p, s);
    case 2 * 32 + 2: return launch_tc_t<2, 2>(p, s);
    case 2 * 32 + 4: return launch_tc_t<2, 4>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

TQ_BOUNDS_READER(bounds_flag_prefill_tc)

}  // namespace tq
