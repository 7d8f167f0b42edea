// Tensor-core decode attention on the packed cache ([TQ] 四-六; [AQJL] QJL).
//
// Why tensor cores: per cached token a GQA group of G = 4 query heads needs
// 4 x (256 + 128) sign/plane products plus 4 x 128 P V products; on CUDA cores
// that is several times the instruction budget of streaming 120 bytes per
// token at HBM speed.  Both contractions are dense (tokens x features x heads),
// so they run on warp-level MMA:
//
//   logits  int8 mma.sync m16n8k32: A = key feature bits of 16 tokens as u8,
//           one AND per 4 bits: the stored bit of MMA index k sits at bit t of
//           its byte (t = (k mod 16) / 4, + 4 for k >= 16), so the masked byte
//           is 2^t or 2^(4+t); B = the query weights in 24-bit fixed point,
//           times 2^(7-t) (resp. 2^(3-t)) so that every product carries the
//           same 2^7, as four signed int8 slices (the two n-tiles hold the four
//           slices of the four heads); the integer accumulation is exact.
//           For a symmetric Lloyd-Max
//           codebook c[idx] = sum over odd bit-subsets S of w_S (-1)^{xor of
//           the bits in S} (a Walsh expansion whose even terms vanish), so the
//           MSE term is linear in the stored bit-planes:
//             <Pi q, c[idx]> = (sum_S w_S)(sum_j qr_j) - 2 sum_S w_S sum_j qr_j x_Sj.
//           The QJL term uses <qs, 2 s - 1> = 2 <qs, s> - sum qs.
//   P V     f16 mma.sync m16n8k16: A = value codes (channels x tokens) as f16
//           code * 2^(2k-24), k the code's place in its byte: the cache keeps
//           the codes of a token pair interleaved by 16-bit halves, so one AND
//           of a stored word (shifted by a byte for half of the lanes) is the
//           operand of two tokens (the per-channel power of two is undone once
//           per split); B = p * s split into f16 hi + lo (the value scale s is
//           per token and group).
//
// One CTA = one (batch, KV head, split) with 4 warps; the two warp pairs take
// alternate blocks and each warp owns 32 of the 64 tokens of its pair's blocks
// (two m-tiles) and keeps its own online-softmax state; blocks are
// staged in shared memory by cp.async.bulk with mbarrier completion (4 stages,
// bounded waits that raise an error flag instead of hanging).  The last split
// also folds in the exact ring tokens.  Warps merge at the end; the split's
// (m, l, o) goes to the same workspace the combine kernel reads.
//
// Specialisation: head dim 128, G = 4, 2-bit values in groups of 32, b1 in
// {0, 1, 2}, m in {64, 128, 192, 256, 384, 512}.  Other shapes use
// decode_kernels.cu.
#include <cfloat>

#include "mma_common.cuh"
#include "prep_mma.cuh"

namespace tq {
namespace {
using namespace mmadec;

constexpr int MD = 128;          // head dim of this path
constexpr int NST = 4;           // pipeline stages (blocks in flight per CTA)
constexpr int MT = 128;          // threads per CTA
constexpr int kPairBytes = 2 * MD * 2 / 8;   // value codes of a token pair (2-bit)
// Workspace views used here: per (batch, KV head) unit, fragment words
// [kstep][lane][ntile][reg] (uint32) and per head {kM, CM, kQ, CQ} (float).

// ---------------------------------------------------------------- prep
template <int NV>
__global__ void __launch_bounds__(256) k_prep_mma(Geom g, const void* Q, int Hq, const float* Pi,
                                                  const float* S, const float* cent,
                                                  float scale_log2, DecodeWs ws) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_launch_dependents();   // the partial kernel may launch; it waits for this grid
  prep_mma_body<NV>(g, Q, Hq, Pi, S, cent, scale_log2, ws, blockIdx.x >> 1, blockIdx.x & 1, smem_raw);
}

// ---------------------------------------------------------------- partial
template <int B1, int KSQ>
__global__ void __launch_bounds__(MT, 4) k_decode_partial_mma(MParams p) {
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;
  constexpr int KSM = F * MD / 32;
  constexpr int KS = KSM + KSQ;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[NST];
  __shared__ int s_abort;
  __shared__ float s_m[4][MG], s_l[4][MG];
  __shared__ float s_mn[4][MG][4];
  __shared__ int s_iss[NST];       // copies issued into each stage (for the error-path drain)
  __shared__ __align__(16) uint32_t s_frag[KS * 128];
  __shared__ __align__(8) uint64_t ringbar;
  __shared__ __align__(16) float s_qf[MG * MD];

  const Geom& g = p.g;
  const int split = blockIdx.x, unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int bq0 = b * p.Hq + h * MG;
  const int bb = (int)g.block_bytes;
  unsigned char* stage = smem_raw;                       // [NST][bb]
  float* s_out = reinterpret_cast<float*>(smem_raw + (size_t)NST * bb);   // [4][MG][MD]

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
  const uint8_t* region = p.base + (int64_t)unit * g.region_bytes;

  // The exact ring tokens are folded in by the last split, a chunk of RC of them at
  // a time staged in the (until the final merge unused) s_out area; the first chunk
  // is requested here, before the cache blocks.
  const bool ring_split = split == p.splits - 1 && p.n_ring > 0;
  const int es = g.dtype == TQ_F32 ? 4 : 2;
  const int RC = (4 * MG * MD * (int)sizeof(float)) / (2 * MD * es);
  const unsigned char* ring_k = p.base + g.ring_k_off + (int64_t)unit * g.W * MD * es;
  const unsigned char* ring_v = p.base + g.ring_v_off + (int64_t)unit * g.W * MD * es;
  unsigned char* s_rk = reinterpret_cast<unsigned char*>(s_out);
  unsigned char* s_rv = s_rk + (size_t)RC * MD * es;
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
    mbar_init(&ringbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Launched programmatically after the preparation kernel (or the fused quantise
  // and preparation of a decode step): of what that grid may write, only the packed
  // blocks below p.early_blk are touched before the wait for it, where they fill
  // the first stages while it runs.
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) s_iss[s] = 0;
    for (int s = 0; s < NST && s < nb && blk0 + s < p.early_blk; ++s) {
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s], p.base, g.total_bytes, 107);
      s_iss[s] = 1;
    }
  }
  pdl_wait();
  if (tid == 0) {
    if (ring_split) {
      const uint32_t nbytes = (uint32_t)(min(RC, p.n_ring) * MD * es);
      mbar_expect_tx(&ringbar, 2 * nbytes);
      cache_bulk_load(s_rk, ring_k, nbytes, &ringbar, p.base, g.total_bytes, 101);
      cache_bulk_load(s_rv, ring_v, nbytes, &ringbar, p.base, g.total_bytes, 102);
    }
    for (int s = 0; s < NST && s < nb; ++s) {
      if (s_iss[s]) continue;
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s], p.base, g.total_bytes, 103);
      s_iss[s] = 1;
    }
  }
  if (ring_split)
    for (int i = tid; i < MG * MD; i += MT) s_qf[i] = p.ws.qf[(int64_t)bq0 * MD + i];

  // B fragments of the score (query slices), per k-step and lane four words
  // {ntile0 r0, ntile0 r1, ntile1 r0, ntile1 r1}, staged in shared memory.
  {
    const uint4* fr = reinterpret_cast<const uint4*>(p.ws.frag + (int64_t)unit * (KS * 128));
    for (int i = tid; i < KS * 32; i += MT) reinterpret_cast<uint4*>(s_frag)[i] = fr[i];
  }
  const float* qc = p.ws.qconst + ((int64_t)unit * MG + tig) * 4;
  const float kM = qc[0], CM = qc[1], kQ = qc[2], CQ = qc[3];
  __syncthreads();
  const uint4* bfr = reinterpret_cast<const uint4*>(s_frag) + lane;

  const uint32_t maskA = 0x01010101u << tig, maskB = 0x10101010u << tig;
  // P V rows: row gid (h = 0) and gid + 8 (h = 1) of m-tile mt = 2 gi + e are the
  // channels 32 gi + 4 gid + 2 e + h: byte gid & 1, code 2 e + h of that byte, of
  // the 16-bit half s = gid >> 1 of value group gi.  A word of a token-pair record
  // (even token low, odd token high) shifted right by 8 (gid & 1) and masked with
  // 0x00030003 << 2k (k = 2 e + h) is the f16x2 operand code * 2^(2k - 24) of both
  // tokens (raw values below 2^10: exact subnormals).
  const uint32_t vshift = 8u * (uint32_t)(gid & 1);
  const int vc_lane = 16 * (gid >> 1);        // byte of this lane's four words in a pair record

  float m_run = -INFINITY, l_run = 0.f;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
  float mnacc[4] = {0.f, 0.f, 0.f, 0.f};
  const bool odd = (gid & 1) != 0;
  const float oddf = odd ? 1.f : 0.f;
  const int hP = gid >> 1;

  // One 16-token step of this warp: logits l0 (token row gid) / l1 (row gid+8) for
  // head tig are given; returns p0, p1 relative to the running max of the head.
  // The running max is raised (with a reduction over the warp and a rescale of
  // the accumulators) only when a logit exceeds it by more than kLazy (log2
  // units), so p <= 2^kLazy; the running sum is kept per lane and reduced once.
  constexpr float kLazy = 4.f;
  // Raise the running max of head tig to at least the warp's max of lmax over gid,
  // rescaling the running sum and the accumulators.
  auto raise_max = [&](float lmax) {
    {
      float mx = lmax;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run, mx);
      const float alpha = (m_run == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f)
                                               : exp2f(m_run - m_new);
      m_run = m_new;
      l_run *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] *= alpha;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) mnacc[gi] *= alpha;       // head tig, like m_run
    }
  };
  auto softmax_step = [&](float l0, float l1, float& p0, float& p1) {
    const float lmax = fmaxf(l0, l1);
    if (__any_sync(0xffffffffu, lmax > m_run + kLazy)) raise_max(lmax);
    if (m_run == -INFINITY) {
      p0 = 0.f;
      p1 = 0.f;
    } else {
      p0 = exp2f(l0 - m_run);
      p1 = exp2f(l1 - m_run);
    }
    l_run += p0 + p1;
  };

  // Warp w takes the blocks j = (w >> 1) (mod 2) of this split (stages alternate
  // between the two warp pairs, NST even) and, in each, the 32 tokens
  // 32 (w & 1) .. +31 as two 16-token m-tiles.
  const int pair = warp >> 1, tb = 32 * (warp & 1);
  for (int j = pair; j < nb; j += 2) {
    const int st = j % NST;
    const uint32_t phase = (uint32_t)((j / NST) & 1);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], phase));
    if (!ok) {
      if (lane == 0) {
        atomicExch(p.err, 1);
        s_abort = 1;
      }
    }
    if (ok) {
    const unsigned char* blk = stage + (size_t)st * bb;
    const int64_t tok0 = (blk0 + j) * kBlockTokens;
    const int nt_valid = (int)min((int64_t)kBlockTokens, p.n_comp - tok0);

    // ---------------- logits of tokens tb + 16 r + gid + 8 e (r, e in {0, 1})
    float vM[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, vQ[2][2];
    if constexpr (KSM > 0) {
      int a[2][2][4] = {};   // [m-tile][ntile][4]
#pragma unroll
      for (int c = 0; c < KSM; c += 4) {
        uint32_t w[2][2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            lds_words<4>(blk + g.o_idx + (tb + 16 * r + gid + 8 * e) * (KSM * 4) + 4 * c, w[r][e]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint4 bq = bfr[(c + kk) * 32];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const uint32_t a0 = w[r][0][kk] & maskA, a1 = w[r][1][kk] & maskA;
            const uint32_t a2 = w[r][0][kk] & maskB, a3 = w[r][1][kk] & maskB;
            imma16832(a[r][0], a0, a1, a2, a3, bq.x, bq.y);
            imma16832(a[r][1], a0, a1, a2, a3, bq.z, bq.w);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) vM[r][e] = slices_to_float(a[r][0][2 * e], a[r][0][2 * e + 1],
                                                               a[r][1][2 * e], a[r][1][2 * e + 1]);
    }
    {
      constexpr int CQ4 = KSQ % 4 == 0 ? 4 : 2;       // words per shared-memory load
      int a[2][2][4] = {};
#pragma unroll
      for (int c = 0; c < KSQ; c += CQ4) {
        uint32_t w[2][2][CQ4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            lds_words<CQ4>(blk + g.o_sign + (tb + 16 * r + gid + 8 * e) * (KSQ * 4) + 4 * c, w[r][e]);
#pragma unroll
        for (int kk = 0; kk < CQ4; ++kk) {
          const uint4 bq = bfr[(KSM + c + kk) * 32];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const uint32_t a0 = w[r][0][kk] & maskA, a1 = w[r][1][kk] & maskA;
            const uint32_t a2 = w[r][0][kk] & maskB, a3 = w[r][1][kk] & maskB;
            imma16832(a[r][0], a0, a1, a2, a3, bq.x, bq.y);
            imma16832(a[r][1], a0, a1, a2, a3, bq.z, bq.w);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) vQ[r][e] = slices_to_float(a[r][0][2 * e], a[r][0][2 * e + 1],
                                                               a[r][1][2 * e], a[r][1][2 * e + 1]);
    }
    const float* rho = reinterpret_cast<const float*>(blk + g.o_rho);
    const float* rn = reinterpret_cast<const float*>(blk + g.o_rnorm);
    float l[2][2];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = tb + 16 * r + gid + 8 * e;
        float v = B1 > 0 ? rho[t] * fmaf(kM, vM[r][e], CM) + rn[t] * fmaf(kQ, vQ[r][e], CQ)
                         : rho[t] * fmaf(kQ, vQ[r][e], CQ);
        if (nt_valid < kBlockTokens && t >= nt_valid) v = -INFINITY;
        l[r][e] = v;
      }
    if (p.logits) {
      const float inv = 1.f / p.scale_log2;
      float* lg = p.logits + (int64_t)(bq0 + tig) * p.n_log + tok0;
      const int64_t nlog_all = (int64_t)g.B * p.Hq * p.n_log;
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = tb + 16 * r + gid + 8 * e;
          if (t < nt_valid && TQ_CHECKED(lg + t, 4, p.logits, 4 * nlog_all, 111)) lg[t] = l[r][e] * inv;
        }
    }

    // ---------------- softmax (lazy running max, see softmax_step)
    float pr[2][2];
    {
      const float lmax = fmaxf(fmaxf(l[0][0], l[0][1]), fmaxf(l[1][0], l[1][1]));
      if (__any_sync(0xffffffffu, lmax > m_run + kLazy)) raise_max(lmax);
      if (m_run == -INFINITY) {
        pr[0][0] = pr[0][1] = pr[1][0] = pr[1][1] = 0.f;
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e) pr[r][e] = exp2f(l[r][e] - m_run);
      }
      l_run += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
      // the value minima enter as sum_t p_t mn_{t,g} per head (tig) and group
      const float4* vm4 = reinterpret_cast<const float4*>(blk + g.o_vmin);
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4 mv = vm4[tb + 16 * r + gid + 8 * e];
          mnacc[0] = fmaf(pr[r][e], mv.x, mnacc[0]);
          mnacc[1] = fmaf(pr[r][e], mv.y, mnacc[1]);
          mnacc[2] = fmaf(pr[r][e], mv.z, mnacc[2]);
          mnacc[3] = fmaf(pr[r][e], mv.w, mnacc[3]);
        }
    }

    // ---------------- P V, one 16-token m-tile at a time
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      // MMA indices k = 2tig, 2tig+1 of this lane are the m-tile's tokens TA = 2tig,
      // TB = 2tig+1 (token pair tig), k = 2tig+8, 2tig+9 are TC = TA+8, TD = TA+9
      // (pair tig+4); their p (head hP) come from the score lanes gid = 2tig, 2tig+1
      // (rows e = 0 for TA, TB and e = 1 for TC, TD).
      const float pA = __shfl_sync(0xffffffffu, pr[r][0], 8 * tig + hP);
      const float pB = __shfl_sync(0xffffffffu, pr[r][0], 8 * tig + 4 + hP);
      const float pC = __shfl_sync(0xffffffffu, pr[r][1], 8 * tig + hP);
      const float pD = __shfl_sync(0xffffffffu, pr[r][1], 8 * tig + 4 + hP);
      const int TA = tb + 16 * r + 2 * tig, TB = TA + 1, TC = TA + 8, TD = TA + 9;
      const float4* vs4 = reinterpret_cast<const float4*>(blk + g.o_vscale);
      const float4 sA = vs4[TA], sB = vs4[TB], sC = vs4[TC], sD = vs4[TD];
      uint32_t bpv[4][2];
      {
        const float sa[4] = {sA.x, sA.y, sA.z, sA.w}, sb[4] = {sB.x, sB.y, sB.z, sB.w};
        const float sc[4] = {sC.x, sC.y, sC.z, sC.w}, sd[4] = {sD.x, sD.y, sD.z, sD.w};
        const float2 pAB = make_float2(pA, pB), pCD = make_float2(pC, pD);
        const float2 nodd = make_float2(-oddf, -oddf);
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          // tokens past the end have p = 0 and finite (zeroed or earlier) metadata
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
      // this lane's words (s = gid >> 1, groups 0..3) of the pairs tig and tig + 4
      const unsigned char* vc = blk + g.o_vcode + vc_lane;
      const uint4 wAB = *reinterpret_cast<const uint4*>(vc + (TA >> 1) * kPairBytes);
      const uint4 wCD = *reinterpret_cast<const uint4*>(vc + (TC >> 1) * kPairBytes);
      const uint32_t ab[4] = {wAB.x >> vshift, wAB.y >> vshift, wAB.z >> vshift, wAB.w >> vshift};
      const uint32_t cd[4] = {wCD.x >> vshift, wCD.y >> vshift, wCD.z >> vshift, wCD.w >> vshift};
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int gi = mt >> 1;
        const uint32_t m0 = 0x00030003u << (4 * (mt & 1)), m1 = m0 << 2;
        hmma16816(acc[mt], ab[gi] & m0, ab[gi] & m1, cd[gi] & m0, cd[gi] & m1, bpv[gi][0],
                  bpv[gi][1]);
      }
    }
    }  // ok
    // Release the stage: the two warps of the pair meet at their named barrier,
    // which also ORs their view of the abort flag (so that both leave the loop
    // together and every barrier is met by both); then the pair's first warp
    // refills the stage with block j + NST (same parity, so the same pair
    // consumes it).
    if (pair_release(pair, *((volatile int*)&s_abort) != 0)) break;
    if ((warp & 1) == 0 && lane == 0 && j + NST < nb) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&full[st], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)st * bb, region + (blk0 + j + NST) * bb, (uint32_t)bb,
                &full[st], p.base, g.total_bytes, 104);
      s_iss[st] += 1;
    }
  }
  __syncthreads();

  if (s_abort) {
    // a wait gave up: wait (bounded) for the last copy issued into every stage,
    // then leave
    if (tid == 0) {
      for (int s = 0; s < NST; ++s)
        if (s_iss[s] > 0) (void)mbar_wait(&full[s], (uint32_t)((s_iss[s] - 1) & 1));
      if (ring_split) (void)mbar_wait(&ringbar, 0);
    }
    return;
  }

  // ---------------- exact ring tokens (last split)
  // acc[mt][c] is channel 32 (mt >> 1) + 4 gid + 2 (mt & 1) (+1 for c >= 2) of head
  // tig in units of 2^(2k - 24), k = 2 (mt & 1) (+1 for c >= 2).
  auto code_unit = [&](int mt) {      // 2^(2k - 24) of row gid; row gid + 8: times 4
    return __int_as_float((127 - 24 + 4 * (mt & 1)) << 23);
  };
  auto chan = [&](int mt) { return 32 * (mt >> 1) + 4 * gid + 2 * (mt & 1); };
  if (ring_split) {
    // Ring slots in slot order (softmax and P V do not depend on the order); slot s
    // holds the token at ring position ((s - first) mod W).  Warp w takes the slots
    // per_warp * w + (0 .. per_warp-1) of each chunk as its rows gid < per_warp.
    const int64_t first = p.n_total - p.n_ring;
    const int per_warp = RC / 4;
    for (int c0 = 0, ci = 0; c0 < p.n_ring; c0 += RC, ++ci) {
      const int nc = min(RC, p.n_ring - c0);
      if (ci > 0 && tid == 0) {
        const uint32_t nbytes = (uint32_t)(nc * MD * es);
        mbar_expect_tx(&ringbar, 2 * nbytes);
        cache_bulk_load(s_rk, ring_k + (int64_t)c0 * MD * es, nbytes, &ringbar, p.base, g.total_bytes, 105);
        cache_bulk_load(s_rv, ring_v + (int64_t)c0 * MD * es, nbytes, &ringbar, p.base, g.total_bytes, 106);
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&ringbar, (uint32_t)(ci & 1)));
      if (!ok && lane == 0) {
        atomicExch(p.err, 1);
        s_abort = 1;
      }
      __syncthreads();
      if (s_abort) {
        if (tid == 0) (void)mbar_wait(&ringbar, (uint32_t)(ci & 1));
        return;
      }
      const int sl = per_warp * warp + gid;
      float l = -INFINITY;
      if (gid < per_warp && sl < nc) {
        const float* q = s_qf + tig * MD;
        float dot = 0.f;
#pragma unroll 8
        for (int j = 0; j < MD; ++j) dot = fmaf(q[j], load_f(s_rk, (int64_t)sl * MD + j, g.dtype), dot);
        const int64_t rt = ((int64_t)(c0 + sl) - first % g.W + g.W) % g.W;
        float* dst = p.logits + (int64_t)(bq0 + tig) * p.n_log + p.n_comp + rt;
        if (p.logits && TQ_CHECKED(dst, 4, p.logits, 4 * (int64_t)g.B * p.Hq * p.n_log, 112))
          *dst = dot;
        l = dot * p.scale_log2;
      }
      float p0, p1;
      softmax_step(l, -INFINITY, p0, p1);
      // column 2 tig + (c & 1) of acc is head tig: add p * v into the hi column (c
      // even) in code units
      for (int T = 0; T < per_warp; ++T) {
        const float pt = __shfl_sync(0xffffffffu, p0, 4 * T + tig);
        const int sl2 = per_warp * warp + T;
        if (sl2 >= nc) break;
        const int64_t e = (int64_t)sl2 * MD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const float v0 = load_f(s_rv, e + chan(mt), g.dtype);
          const float v1 = load_f(s_rv, e + chan(mt) + 1, g.dtype);
          const float u = code_unit(mt);
          acc[mt][0] = fmaf(pt * v0, u, acc[mt][0]);
          acc[mt][2] = fmaf(pt * v1, 4.f * u, acc[mt][2]);
        }
      }
      __syncthreads();     // the chunk is consumed before the next one is requested
    }
  }

  // ---------------- merge the 4 warps
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  if (gid == 0) {
    s_m[warp][tig] = m_run;
    s_l[warp][tig] = l_run;
  }
  // mn sums of head tig: reduce over gid
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    float v = mnacc[gi];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    if (gid == 0) s_mn[warp][tig][gi] = v;
  }
  __syncthreads();
  // this lane's channels, head tig: o = code part (hi + lo) + mn part, scaled to the CTA max
  float Mh = -INFINITY;
  for (int w = 0; w < 4; ++w) Mh = fmaxf(Mh, s_m[w][tig]);
  const float sc = (m_run == -INFINITY) ? 0.f : exp2f(m_run - Mh);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const float mnv = s_mn[warp][tig][mt >> 1];
    const float inv = __int_as_float((127 + 24 - 4 * (mt & 1)) << 23);   // 1 / code_unit(mt)
    const float o0 = ((acc[mt][0] + acc[mt][1]) * inv + mnv) * sc;
    const float o1 = ((acc[mt][2] + acc[mt][3]) * (0.25f * inv) + mnv) * sc;
    *reinterpret_cast<float2*>(&s_out[(warp * MG + tig) * MD + chan(mt)]) = make_float2(o0, o1);
  }
  __syncthreads();
  const int64_t rows = (int64_t)g.B * p.Hq;
  for (int i = tid; i < MG * MD; i += MT) {
    const int hh = i / MD, ch = i % MD;
    float o = 0.f;
    for (int w = 0; w < 4; ++w) o += s_out[(w * MG + hh) * MD + ch];
    float* dst = p.ws.part_o + ((int64_t)(bq0 + hh) * p.splits + split) * MD + ch;
    if (TQ_CHECKED(dst, 4, p.ws.part_o, 4 * rows * p.splits * MD, 113)) *dst = o;
  }
  if (tid < MG) {
    float M = -INFINITY, L = 0.f;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w][tid]);
    if (M != -INFINITY)
      for (int w = 0; w < 4; ++w)
        if (s_m[w][tid] != -INFINITY) L += s_l[w][tid] * exp2f(s_m[w][tid] - M);
    float* dst = p.ws.part_ml + ((int64_t)(bq0 + tid) * p.splits + split) * 2;
    if (TQ_CHECKED(dst, 8, p.ws.part_ml, 8 * rows * p.splits, 114)) {
      dst[0] = M;
      dst[1] = L;
    }
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
    merge_splits<MD, MT>(p, bq0);
    return;
  }
  for (int i = tid; i < MG * MD; i += MT) {
    const int hh = i / MD, ch = i % MD;
    const int bq = bq0 + hh;
    const volatile float* ml = p.ws.part_ml + (int64_t)bq * p.splits * 2;
    const volatile float* po = p.ws.part_o + (int64_t)bq * p.splits * MD;
    float M = -INFINITY;
    for (int sp = 0; sp < p.splits; ++sp) M = fmaxf(M, ml[2 * sp]);
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
      for (int sp = 0; sp < p.splits; ++sp) {
        const float ms = ml[2 * sp];
        if (ms == -INFINITY) continue;
        const float wgt = exp2f(ms - M);
        L = fmaf(ml[2 * sp + 1], wgt, L);
        o = fmaf(po[sp * MD + ch], wgt, o);
      }
      o = o / L;
    }
    if (TQ_CHECKED((const char*)p.out + ((int64_t)bq * MD + ch) * es, es, p.out, rows * MD * es, 115))
      store_f(p.out, (int64_t)bq * MD + ch, g.dtype, o);
  }
}

template <int B1, int KSQ>
cudaError_t launch_partial_t(const MParams& p, cudaStream_t s) {
  const size_t smem = (size_t)NST * p.g.block_bytes + sizeof(float) * 4 * MG * MD;
  cudaError_t e = cudaFuncSetAttribute(k_decode_partial_mma<B1, KSQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.splits, (unsigned)(p.g.B * p.g.Hkv));
  return launch_pdl(k_decode_partial_mma<B1, KSQ>, grid, dim3(MT), smem, s, p);
}

}  // namespace

bool decode_mma_supported(const Geom& g, int G) {
  if (decode_wide_supported(g, G)) return true;
  return g.d == MD && G == MG && g.vbits == 2 && g.group == 32 && g.b1 <= 2 &&
         (g.m == 64 || g.m == 128 || g.m == 192 || g.m == 256 || g.m == 384 || g.m == 512);
}

int decode_mma_ctas_per_sm(const Geom& g) { return g.d == 256 ? 2 : 4; }

cudaError_t launch_decode_prep_mma(const Geom& g, const void* Q, int Hq, const float* Pi,
                                   const float* S, const float* cent, float scale,
                                   const DecodeWs& ws, cudaStream_t s) {
  const size_t smem = prep_smem_bytes(g.d, g.m);
  auto kern = g.d == 256 ? k_prep_mma<2> : k_prep_mma<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<2 * g.B * g.Hkv, 256, smem, s>>>(g, Q, Hq, Pi, S, cent, scale * kLog2e, ws);   // 2 halves a unit
  return cudaGetLastError();
}

cudaError_t launch_decode_partial_mma(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                      float scale, float* logits, int splits, const DecodeWs& ws,
                                      void* out, int64_t early_blk, cudaStream_t s) {
  MParams p{};
  p.out = out;
  p.early_blk = early_blk;
  p.g = g;
  p.base = base;
  p.n_total = n_total;
  p.n_comp = n_total > g.W ? n_total - g.W : 0;
  p.n_ring = (int)(n_total < g.W ? n_total : g.W);
  p.Hq = Hq;
  p.scale_log2 = scale * kLog2e;
  p.logits = logits;
  p.n_log = p.n_comp + p.n_ring;
  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  p.splits = splits;
  p.bps = (int)((nblk + splits - 1) / splits);
  p.ws = ws;
  p.err = ws.err;
  if (g.d == 256) return launch_partial_wide(p, s);
  const int ksq = g.m / 32;
  switch (g.b1 * 32 + ksq) {
    case 0 * 32 + 2: return launch_partial_t<0, 2>(p, s);
    case 0 * 32 + 4: return launch_partial_t<0, 4>(p, s);
    case 0 * 32 + 6: return launch_partial_t<0, 6>(p, s);
    case 0 * 32 + 8: return launch_partial_t<0, 8>(p, s);
    case 0 * 32 + 12: return launch_partial_t<0, 12>(p, s);
    case 0 * 32 + 16: return launch_partial_t<0, 16>(p, s);
    case 1 * 32 + 2: return launch_partial_t<1, 2>(p, s);
    case 1 * 32 + 4: return launch_partial_t<1, 4>(p, s);
    case 1 * 32 + 6: return launch_partial_t<1, 6>(p, s);
    case 1 * 32 + 8: return launch_partial_t<1, 8>(p, s);
    case 1 * 32 + 12: return launch_partial_t<1, 12>(p, s);
    case 1 * 32 + 16: return launch_partial_t<1, 16>(p, s);
    case 2 * 32 + 2: return launch_partial_t<2, 2>(p, s);
    case 2 * 32 + 4: return launch_partial_t<2, 4>(p, s);
    case 2 * 32 + 6: return launch_partial_t<2, 6>(p, s);
    case 2 * 32 + 8: return launch_partial_t<2, 8>(p, s);
    case 2 * 32 + 12: return launch_partial_t<2, 12>(p, s);
    case 2 * 32 + 16: return launch_partial_t<2, 16>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

TQ_BOUNDS_READER(bounds_flag_decode_mma)

}  // namespace tq
