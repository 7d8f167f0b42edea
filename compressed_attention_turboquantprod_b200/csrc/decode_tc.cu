// Decode attention on the packed cache with the score contraction on the
// fifth-generation tensor cores ([TQ] 四-六; [AQJL] QJL).  Head dim 128, G = 4
// query heads per KV head, 2-bit values in groups of 32, b1 in {0, 1, 2},
// m in {64, 128, 192, 256, 384, 512}.
//
// The logit of a cached token is linear in its stored bits: for a symmetric
// Lloyd-Max codebook c[idx] is a Walsh sum over odd bit-subsets, so
//   <Pi q, c[idx]> = (sum_S w_S)(sum_j qr_j) - 2 sum_S w_S sum_j qr_j x_Sj
// with x_Sj the stored feature bits, and the QJL term is <qs, 2 s - 1>.  A
// 128-token chunk (two cache blocks) is one tcgen05.mma.kind::i8 problem:
//   D[128 tokens x 16] = A[128 tokens x K] . B[K x 16]
// A = the tokens' feature bits as unsigned bytes, written by each token's own
// thread straight into tensor memory (the A-from-tensor-memory form: the
// expanded operand never touches shared memory).  Column 8k + t of k-step k
// holds the stored word k of the token masked with 0x01010101 << t, so byte b
// of that column is bit t of stored byte b, i.e. feature 32k + 8b + t, with
// value 2^t.  B = the query weights in 24-bit fixed point times 2^(7-t), four
// signed int8 slices per head (16 columns: column 4h + slice), in shared
// memory (canonical K-major layout without swizzle).  The integer
// accumulation in tensor memory is exact; the MSE and QJL k-steps accumulate
// into separate 16-column accumulators because they take different per-token
// factors (rho and ||r||).  One thread issues the MMAs and commits them to an
// mbarrier.
//
// Each thread then reads its token's 32 accumulator columns, forms the logits
// of the four heads, and feeds a per-warp online softmax (lazy running max).
// P V stays on warp-level MMA (f16 m16n8k16, value codes as f16 subnormals
// from the token-pair records, B = p * s split into f16 hi + lo): its operands
// come from 2-bit codes and per-token scales, which the register-fed form
// consumes without an expanded copy.
//
// One CTA = one (batch, KV head, split), 4 warps; warp w owns tokens
// 32 (w & 1) .. +31 of block 2c + (w >> 1) of chunk c (its tensor-memory lanes
// 32 w .. 32 w + 31).  Cache blocks arrive by cp.async.bulk into 4 shared-memory
// stages with mbarrier completion; every wait is bounded (error flag, drain of
// the copies in flight, tensor memory freed; never a hang).  The last split
// folds in the exact ring tokens, and the last split of a unit to finish merges
// the splits and writes the output.
#include <cfloat>

#include "mma_common.cuh"
#include "tc_common.cuh"

namespace tq {
namespace mmadec {
namespace {

constexpr int MD = 128;             // head dim of this path
constexpr int NST = 4;              // block stages (a chunk takes two)
constexpr int MT = 128;             // threads per CTA
constexpr int KA = 12;              // k-steps of A held in tensor memory at a time
constexpr uint32_t kTmemCols = 128; // A: KA * 8 = 96 columns; D: 32 columns
constexpr uint32_t kColD = KA * 8;  // D_MSE at kColD .. +15, D_QJL at kColD + 16 .. +31
constexpr int kPairBytes = 2 * MD * 2 / 8;   // value codes of a token pair (2-bit)
constexpr int kBKStep = 512;        // shared-memory bytes of B per k-step (16 rows x 32 bytes)

// kind::i8 instruction descriptor: s32 D, u8 A, s8 B, both K-major, M = 128, N = 16.
constexpr uint32_t kIdescI8 =
    (2u << 4) | (0u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory descriptor of B: 8-row x 16-byte core matrices, the two K halves
// of a k-step 128 bytes apart (leading byte offset), the two 8-row groups 256
// bytes apart (stride byte offset), no swizzle, descriptor version 1.
__device__ __forceinline__ uint64_t bdesc_i8(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
         ((uint64_t)(256 >> 4) << 32) | (1ull << 46);
}

// D[tmem] (+)= A[tmem] . B[smem]^T, kind::i8, issued by one thread.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %4, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(accumulate), "r"(kIdescI8)
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane (warp-wide).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
        "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]),
        "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
        "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// The eight masked words (features 32k + 8b + t, value 2^t) of one stored word.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t* o) {
#pragma unroll
  for (int t = 0; t < 8; ++t) o[t] = w & (0x01010101u << t);
}

template <int B1, int KSQ>
__global__ void __launch_bounds__(MT, 4) k_decode_partial_tc(MParams p) {
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;
  constexpr int KSM = F * MD / 32;          // MSE k-steps (feature planes x 4)
  constexpr int KS = KSM + KSQ;
  constexpr int NPASS = (KS + KA - 1) / KA;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[NST];
  __shared__ __align__(8) uint64_t mmabar;
  __shared__ __align__(8) uint64_t ringbar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_cnt[NST];
  __shared__ int s_iss[NST];
  __shared__ float s_m[4][MG], s_l[4][MG];
  __shared__ float s_mn[4][MG][4];
  __shared__ __align__(16) float s_qc[MG * 4];          // per head {kM, CM, kQ, CQ}
  __shared__ __align__(16) float s_p[4][32][MG];        // p of each warp's tokens
  __shared__ __align__(16) float s_qf[MG * MD];

  const Geom& g = p.g;
  const int split = blockIdx.x, unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int bq0 = b * p.Hq + h * MG;
  const int bb = (int)g.block_bytes;
  unsigned char* stage = smem_raw;                                         // [NST][bb]
  unsigned char* sB = smem_raw + (size_t)NST * bb;                        // [KS][512]
  float* s_out = reinterpret_cast<float*>(sB + (size_t)KS * kBKStep);     // [4][MG][MD]

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
  const uint8_t* region = p.base + (int64_t)unit * g.region_bytes;

  const bool ring_split = split == p.splits - 1 && p.n_ring > 0;
  const int es = g.dtype == TQ_F32 ? 4 : 2;
  const int RC = (4 * MG * MD * (int)sizeof(float)) / (2 * MD * es);
  const unsigned char* ring_k = p.base + g.ring_k_off + (int64_t)unit * g.W * MD * es;
  const unsigned char* ring_v = p.base + g.ring_v_off + (int64_t)unit * g.W * MD * es;
  unsigned char* s_rk = reinterpret_cast<unsigned char*>(s_out);
  unsigned char* s_rv = s_rk + (size_t)RC * MD * es;

  if (warp == 0) {   // tensor memory: the A operand and the two accumulators
    tc::tmem_alloc(smem_u32(&s_tmem), kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
    mbar_init(&mmabar, 1);
    mbar_init(&ringbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Launched programmatically after the preparation kernel: nothing that kernel or
  // an earlier one writes is touched before this wait.
  pdl_wait();
  if (tid == 0) {
    if (ring_split) {
      const uint32_t nbytes = (uint32_t)(min(RC, p.n_ring) * MD * es);
      mbar_expect_tx(&ringbar, 2 * nbytes);
      cache_bulk_load(s_rk, ring_k, nbytes, &ringbar, p.base, g.total_bytes, 101);
      cache_bulk_load(s_rv, ring_v, nbytes, &ringbar, p.base, g.total_bytes, 102);
    }
    for (int s = 0; s < NST; ++s) s_iss[s] = 0;
    for (int s = 0; s < NST && s < nb; ++s) {
      mbar_expect_tx(&full[s], (uint32_t)bb);
      cache_bulk_load(stage + (size_t)s * bb, region + (blk0 + s) * bb, (uint32_t)bb, &full[s],
                      p.base, g.total_bytes, 103);
      s_iss[s] = 1;
    }
  }
  if (ring_split)
    for (int i = tid; i < MG * MD; i += MT) s_qf[i] = p.ws.qf[(int64_t)bq0 * MD + i];
  // B: the query slices of the preparation kernel (word (k, lane, ntile, reg): the
  // four bytes of features 32k + 8i + t, t = tig + 4 reg, of slice 2 ntile +
  // (gid & 1) of head gid >> 1) placed at row n = 4 head + slice, K byte 4t + i.
  {
    const uint32_t* fr = p.ws.frag + (int64_t)unit * (KS * 128);
    for (int wi = tid; wi < KS * 128; wi += MT) {
      const int r = wi & 1, nt = (wi >> 1) & 1, ln = (wi >> 2) & 31, ks = wi >> 7;
      const int gq = ln >> 2, tq = ln & 3;
      const int n = 4 * (gq >> 1) + 2 * nt + (gq & 1);
      const int t = tq + 4 * r;
      const int off = ks * kBKStep + (n >> 3) * 256 + (t >> 2) * 128 + (n & 7) * 16 + 4 * (t & 3);
      *reinterpret_cast<uint32_t*>(sB + off) = fr[wi];
    }
  }
  if (tid < MG * 4) s_qc[tid] = p.ws.qconst[(int64_t)unit * MG * 4 + tid];
  if (tid < NST) s_cnt[tid] = 0;
  tc::fence_async_shared();       // B is read by the tensor core (async proxy)
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t tlane = tmem + ((uint32_t)(32 * warp) << 16);   // this warp's lanes
  const uint32_t sB_addr = smem_u32(sB);

  // per-warp online softmax state: running max per head (log2 units, the same in
  // every lane), per-lane partial sums
  constexpr float kLazy = 4.f;
  float m_run[MG], l_run[MG];
  float mnacc[MG][4];
#pragma unroll
  for (int hh = 0; hh < MG; ++hh) {
    m_run[hh] = -INFINITY;
    l_run[hh] = 0.f;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) mnacc[hh][gi] = 0.f;
  }
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
  const uint32_t vshift = 8u * (uint32_t)(gid & 1);
  const int vc_lane = 16 * (gid >> 1);
  const float oddf = (gid & 1) ? 1.f : 0.f;
  const int hP = gid >> 1;

  // Raise the running maxima to at least the warp's maximum of l[hh] (when the
  // lazy test fired), rescaling sums, minima sums and the P V accumulators.
  auto raise_max = [&](const float (&l)[MG]) {
    float alpha[MG];
#pragma unroll
    for (int hh = 0; hh < MG; ++hh) {
      const float mx = warp_max(l[hh]);
      const float m_new = fmaxf(m_run[hh], mx);
      alpha[hh] = (m_run[hh] == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f)
                                           : exp2f(m_run[hh] - m_new);
      m_run[hh] = m_new;
      l_run[hh] *= alpha[hh];
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) mnacc[hh][gi] *= alpha[hh];
    }
    const float at = tig == 0 ? alpha[0] : tig == 1 ? alpha[1] : tig == 2 ? alpha[2] : alpha[3];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][c] *= at;
  };
  // Online-softmax update with this lane's logits l[hh] (one token): returns p.
  auto softmax_token = [&](const float (&l)[MG], float (&pr)[MG]) {
    bool need = false;
#pragma unroll
    for (int hh = 0; hh < MG; ++hh) need |= l[hh] > m_run[hh] + kLazy;
    if (__any_sync(0xffffffffu, need)) raise_max(l);
#pragma unroll
    for (int hh = 0; hh < MG; ++hh) {
      pr[hh] = m_run[hh] == -INFINITY ? 0.f : exp2f(l[hh] - m_run[hh]);
      l_run[hh] += pr[hh];
    }
  };

  const int pair = warp >> 1, tb = 32 * (warp & 1), tk = tb + lane;
  const int nchunks = (nb + 1) >> 1;
  uint32_t mma_phase = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int j = 2 * c + pair;                 // this warp's block of the chunk
    const bool have = j < nb;
    const int st = j % NST;
    const unsigned char* blk = stage + (size_t)st * bb;
    bool fail = false;
    if (have) fail = !__all_sync(0xffffffffu, mbar_wait(&full[st], (uint32_t)((j / NST) & 1)));

    // ---------------- scores on the tensor cores (NPASS passes of up to KA k-steps)
#pragma unroll 1
    for (int ps = 0; ps < NPASS; ++ps) {
      const int k0 = ps * KA, k1 = min(KS, k0 + KA);
      if (have && !fail) {
#pragma unroll
        for (int kg = 0; kg < KA; kg += 4) {
          const int k = k0 + kg;
          if (k >= k1) break;
          const int nk = min(4, k1 - k);
          uint32_t w[4];
          if (k < KSM) {            // idx planes (KSM is a multiple of 4)
            lds_words<4>(blk + g.o_idx + tk * (KSM * 4) + 4 * k, w);
          } else if constexpr (KSQ % 4 == 0) {
            lds_words<4>(blk + g.o_sign + tk * (KSQ * 4) + 4 * (k - KSM), w);
          } else {
            uint32_t w2[2];
            lds_words<2>(blk + g.o_sign + tk * (KSQ * 4) + 4 * (k - KSM), w2);
            w[0] = w2[0];
            w[1] = w2[1];
            if (nk > 2) {
              lds_words<2>(blk + g.o_sign + tk * (KSQ * 4) + 4 * (k - KSM) + 8, w2);
              w[2] = w2[0];
              w[3] = w2[1];
            } else {
              w[2] = w[3] = 0u;
            }
          }
          if (nk == 4) {
            uint32_t v[32];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) expand_word(w[kk], v + 8 * kk);
            tmem_st32(tlane + 8 * kg, v);
          } else {                  // two k-steps (KSQ = 2 or 6: the tail)
            uint32_t v[16];
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) expand_word(w[kk], v + 8 * kk);
            tmem_st16(tlane + 8 * kg, v);
          }
        }
        tmem_wait_st();
      }
      tc::fence_before_sync();
      if (__syncthreads_or(fail ? 1 : 0)) {
        fail = true;
        break;
      }
      if (tid == 0) {
        tc::fence_after_sync();
        for (int k = k0; k < k1; ++k) {
          const bool mse = k < KSM;
          const uint32_t d = tmem + kColD + (mse ? 0u : 16u);
          mma_i8_ts(d, tmem + 8u * (uint32_t)(k - k0), bdesc_i8(sB_addr + k * kBKStep),
                    (k != 0 && k != KSM) ? 1u : 0u);
        }
        tc::mma_commit(smem_u32(&mmabar));
      }
      const bool ok = mbar_wait(&mmabar, mma_phase);
      mma_phase ^= 1u;
      if (__syncthreads_or(ok ? 0 : 1)) {
        fail = true;
        break;
      }
      tc::fence_after_sync();
    }
    if (fail) {
      if (tid == 0) {
        atomicExch(p.err, 1);
        s_abort = 1;
      }
      break;
    }

    // ---------------- logits of this thread's token (four heads)
    uint32_t dv[32];
    tc::tmem_ld32(tlane + kColD, dv);
    tc::tmem_wait_ld();
    const int64_t tok0 = (blk0 + j) * kBlockTokens;
    const int nt_valid = have ? (int)min((int64_t)kBlockTokens, p.n_comp - tok0) : 0;
    const bool valid = tk < nt_valid;
    float lg[MG];
    {
      const float rho = have ? reinterpret_cast<const float*>(blk + g.o_rho)[tk] : 0.f;
      const float rn = (have && B1 > 0) ? reinterpret_cast<const float*>(blk + g.o_rnorm)[tk] : 0.f;
      const float4* qc4 = reinterpret_cast<const float4*>(s_qc);
#pragma unroll
      for (int hh = 0; hh < MG; ++hh) {
        const float4 qc = qc4[hh];    // kM, CM, kQ, CQ
        const float vQ = slices_to_float((int)dv[16 + 4 * hh], (int)dv[17 + 4 * hh],
                                         (int)dv[18 + 4 * hh], (int)dv[19 + 4 * hh]);
        float v;
        if constexpr (B1 > 0) {
          const float vM = slices_to_float((int)dv[4 * hh], (int)dv[4 * hh + 1],
                                           (int)dv[4 * hh + 2], (int)dv[4 * hh + 3]);
          v = rho * fmaf(qc.x, vM, qc.y) + rn * fmaf(qc.z, vQ, qc.w);
        } else {
          v = rho * fmaf(qc.z, vQ, qc.w);
        }
        lg[hh] = valid ? v : -INFINITY;
      }
    }
    if (p.logits && valid) {
      const float inv = 1.f / p.scale_log2;
      const int64_t nlog_all = (int64_t)g.B * p.Hq * p.n_log;
#pragma unroll
      for (int hh = 0; hh < MG; ++hh) {
        float* dst = p.logits + (int64_t)(bq0 + hh) * p.n_log + tok0 + tk;
        if (TQ_CHECKED(dst, 4, p.logits, 4 * nlog_all, 107)) *dst = lg[hh] * inv;
      }
    }

    // ---------------- softmax; the value minima enter as sum_t p_t mn_{t,g}
    float pr[MG];
    softmax_token(lg, pr);
    if (have) {
      const float4 mv = reinterpret_cast<const float4*>(blk + g.o_vmin)[tk];
#pragma unroll
      for (int hh = 0; hh < MG; ++hh) {
        mnacc[hh][0] = fmaf(pr[hh], mv.x, mnacc[hh][0]);
        mnacc[hh][1] = fmaf(pr[hh], mv.y, mnacc[hh][1]);
        mnacc[hh][2] = fmaf(pr[hh], mv.z, mnacc[hh][2]);
        mnacc[hh][3] = fmaf(pr[hh], mv.w, mnacc[hh][3]);
      }
    }
    *reinterpret_cast<float4*>(&s_p[warp][lane][0]) = make_float4(pr[0], pr[1], pr[2], pr[3]);
    __syncwarp();

    // ---------------- P V, one 16-token m-tile at a time
    if (have) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        // MMA indices k = 2tig, 2tig+1 of this lane are the m-tile's tokens TA = 2tig,
        // TB = 2tig+1 (token pair tig), k = 2tig+8, 2tig+9 are TC = TA+8, TD = TA+9
        const int la = 16 * r + 2 * tig;
        const float pA = s_p[warp][la][hP], pB = s_p[warp][la + 1][hP];
        const float pC = s_p[warp][la + 8][hP], pD = s_p[warp][la + 9][hP];
        const int TA = tb + la, TC = TA + 8;
        const float4* vs4 = reinterpret_cast<const float4*>(blk + g.o_vscale);
        const float4 sA = vs4[TA], sB4 = vs4[TA + 1], sC = vs4[TC], sD = vs4[TC + 1];
        uint32_t bpv[4][2];
        {
          const float sa[4] = {sA.x, sA.y, sA.z, sA.w}, sb[4] = {sB4.x, sB4.y, sB4.z, sB4.w};
          const float sc[4] = {sC.x, sC.y, sC.z, sC.w}, sd[4] = {sD.x, sD.y, sD.z, sD.w};
          const float2 pAB = make_float2(pA, pB), pCD = make_float2(pC, pD);
          const float2 nodd = make_float2(-oddf, -oddf);
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            // tokens past the end have p = 0 and finite (zeroed or earlier) metadata;
            // column gid even carries fp16(x), odd carries fp16(x - fp16(x))
            const float2 x0 = mul2(pAB, make_float2(sa[gi], sb[gi]));
            const float2 x1 = mul2(pCD, make_float2(sc[gi], sd[gi]));
            const float2 f0 = __half22float2(__floats2half2_rn(x0.x, x0.y));
            const float2 f1 = __half22float2(__floats2half2_rn(x1.x, x1.y));
            const float2 l0 = fma2(nodd, f0, x0), l1 = fma2(nodd, f1, x1);
            __half2 h0 = __floats2half2_rn(l0.x, l0.y);
            __half2 h1 = __floats2half2_rn(l1.x, l1.y);
            bpv[gi][0] = *reinterpret_cast<uint32_t*>(&h0);
            bpv[gi][1] = *reinterpret_cast<uint32_t*>(&h1);
          }
        }
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
      // Release the stage: the second warp of the pair to finish it refills it with
      // block j + NST.
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        const int done = atomicAdd(&s_cnt[st], 1);
        if (done == 1) {
          __threadfence_block();
          s_cnt[st] = 0;
          if (j + NST < nb) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_expect_tx(&full[st], (uint32_t)bb);
            cache_bulk_load(stage + (size_t)st * bb, region + (blk0 + j + NST) * bb, (uint32_t)bb,
                            &full[st], p.base, g.total_bytes, 104);
            s_iss[st] += 1;
          }
        }
      }
    }
    __syncwarp();        // s_p is rewritten by the next chunk
  }
  __syncthreads();

  if (s_abort) {
    // a wait gave up: wait (bounded) for the last copy issued into every stage and
    // for the tensor-core work in flight, free the tensor memory, leave
    if (tid == 0) {
      for (int s = 0; s < NST; ++s)
        if (s_iss[s] > 0) (void)mbar_wait(&full[s], (uint32_t)((s_iss[s] - 1) & 1));
      if (ring_split) (void)mbar_wait(&ringbar, 0);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
      tc::fence_after_sync();
      tc::tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  // the tensor memory is no longer read: free it for the next CTA on this SM
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }

  // ---------------- exact ring tokens (last split)
  // acc[mt][c] is channel 32 (mt >> 1) + 4 gid + 2 (mt & 1) (+1 for c >= 2) of head
  // tig in units of 2^(2k - 24), k = 2 (mt & 1) (+1 for c >= 2).
  auto code_unit = [&](int mt) { return __int_as_float((127 - 24 + 4 * (mt & 1)) << 23); };
  auto chan = [&](int mt) { return 32 * (mt >> 1) + 4 * gid + 2 * (mt & 1); };
  if (ring_split) {
    // Ring slots in slot order (softmax and P V do not depend on the order); slot s
    // holds the token at ring position ((s - first) mod W).  Warp w takes slots
    // w, w + 4, ... of each staged chunk, one per lane.
    const int64_t first = p.n_total - p.n_ring;
    for (int c0 = 0, ci = 0; c0 < p.n_ring; c0 += RC, ++ci) {
      const int nc = min(RC, p.n_ring - c0);
      if (ci > 0 && tid == 0) {
        const uint32_t nbytes = (uint32_t)(nc * MD * es);
        mbar_expect_tx(&ringbar, 2 * nbytes);
        cache_bulk_load(s_rk, ring_k + (int64_t)c0 * MD * es, nbytes, &ringbar, p.base,
                        g.total_bytes, 105);
        cache_bulk_load(s_rv, ring_v + (int64_t)c0 * MD * es, nbytes, &ringbar, p.base,
                        g.total_bytes, 106);
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
      const int nmine = (nc - warp + 3) / 4;          // slots warp, warp + 4, ... < nc
      const int sl = warp + 4 * lane;
      float lr[MG];
#pragma unroll
      for (int hh = 0; hh < MG; ++hh) lr[hh] = -INFINITY;
      if (lane < nmine) {
#pragma unroll
        for (int hh = 0; hh < MG; ++hh) {
          const float* q = s_qf + hh * MD;
          float dot = 0.f;
#pragma unroll 8
          for (int jj = 0; jj < MD; ++jj)
            dot = fmaf(q[jj], load_f(s_rk, (int64_t)sl * MD + jj, g.dtype), dot);
          const int64_t rt = ((int64_t)(c0 + sl) - first % g.W + g.W) % g.W;
          if (p.logits) {
            float* dst = p.logits + (int64_t)(bq0 + hh) * p.n_log + p.n_comp + rt;
            if (TQ_CHECKED(dst, 4, p.logits, 4 * (int64_t)g.B * p.Hq * p.n_log, 108)) *dst = dot;
          }
          lr[hh] = dot * p.scale_log2;
        }
      }
      float pr[MG];
      softmax_token(lr, pr);
      *reinterpret_cast<float4*>(&s_p[warp][lane][0]) = make_float4(pr[0], pr[1], pr[2], pr[3]);
      __syncwarp();
      // column 2 tig + (c & 1) of acc is head tig: add p * v into the hi column (c
      // even) in code units
      for (int T = 0; T < nmine; ++T) {
        const float pt = s_p[warp][T][tig];
        const int64_t e = (int64_t)(warp + 4 * T) * MD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const float v0 = load_f(s_rv, e + chan(mt), g.dtype);
          const float v1 = load_f(s_rv, e + chan(mt) + 1, g.dtype);
          const float u = code_unit(mt);
          acc[mt][0] = fmaf(pt * v0, u, acc[mt][0]);
          acc[mt][2] = fmaf(pt * v1, 4.f * u, acc[mt][2]);
        }
      }
      __syncwarp();
      __syncthreads();     // the chunk is consumed before the next one is requested
    }
  }

  // ---------------- merge the 4 warps
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < MG; ++hh) s_m[warp][hh] = m_run[hh];
  }
#pragma unroll
  for (int hh = 0; hh < MG; ++hh) {
    const float l = warp_sum(l_run[hh]);
    if (lane == 0) s_l[warp][hh] = l;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const float v = warp_sum(mnacc[hh][gi]);
      if (lane == 0) s_mn[warp][hh][gi] = v;
    }
  }
  __syncthreads();
  // this lane's channels, head tig: o = code part (hi + lo) + mn part, scaled to the CTA max
  {
    float Mh = -INFINITY;
    for (int w = 0; w < 4; ++w) Mh = fmaxf(Mh, s_m[w][tig]);
    const float mw = s_m[warp][tig];
    const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - Mh);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const float mnv = s_mn[warp][tig][mt >> 1];
      const float inv = __int_as_float((127 + 24 - 4 * (mt & 1)) << 23);   // 1 / code_unit(mt)
      const float o0 = ((acc[mt][0] + acc[mt][1]) * inv + mnv) * sc;
      const float o1 = ((acc[mt][2] + acc[mt][3]) * (0.25f * inv) + mnv) * sc;
      *reinterpret_cast<float2*>(&s_out[(warp * MG + tig) * MD + chan(mt)]) = make_float2(o0, o1);
    }
  }
  __syncthreads();
  const int64_t rows = (int64_t)g.B * p.Hq;
  for (int i = tid; i < MG * MD; i += MT) {
    const int hh = i / MD, ch = i % MD;
    float o = 0.f;
    for (int w = 0; w < 4; ++w) o += s_out[(w * MG + hh) * MD + ch];
    float* dst = p.ws.part_o + ((int64_t)(bq0 + hh) * p.splits + split) * MD + ch;
    if (TQ_CHECKED(dst, 4, p.ws.part_o, 4 * rows * p.splits * MD, 109)) *dst = o;
  }
  if (tid < MG) {
    float M = -INFINITY, L = 0.f;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w][tid]);
    if (M != -INFINITY)
      for (int w = 0; w < 4; ++w)
        if (s_m[w][tid] != -INFINITY) L += s_l[w][tid] * exp2f(s_m[w][tid] - M);
    float* dst = p.ws.part_ml + ((int64_t)(bq0 + tid) * p.splits + split) * 2;
    if (TQ_CHECKED(dst, 8, p.ws.part_ml, 8 * rows * p.splits, 110)) {
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
    if (TQ_CHECKED((const char*)p.out + ((int64_t)bq * MD + ch) * es, es, p.out, rows * MD * es, 111))
      store_f(p.out, (int64_t)bq * MD + ch, g.dtype, o);
  }
}

template <int B1, int KSQ>
cudaError_t launch_tc_t(const MParams& p, cudaStream_t s) {
  constexpr int F = B1 > 0 ? 1 << (B1 - 1) : 0;
  constexpr int KS = F * MD / 32 + KSQ;
  const size_t smem = (size_t)NST * p.g.block_bytes + (size_t)KS * kBKStep +
                      sizeof(float) * 4 * MG * MD;
  cudaError_t e = cudaFuncSetAttribute(k_decode_partial_tc<B1, KSQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.splits, (unsigned)(p.g.B * p.g.Hkv));
  return launch_pdl(k_decode_partial_tc<B1, KSQ>, grid, dim3(MT), smem, s, p);
}

}  // namespace

cudaError_t launch_partial_tc(const MParams& p, cudaStream_t s) {
  const int ksq = p.g.m / 32;
  switch (p.g.b1 * 32 + ksq) {
    case 0 * 32 + 2: return launch_tc_t<0, 2>(p, s);
    case 0 * 32 + 4: return launch_tc_t<0, 4>(p, s);
    case 0 * 32 + 6: return launch_tc_t<0, 6>(p, s);
    case 0 * 32 + 8: return launch_tc_t<0, 8>(p, s);
    case 0 * 32 + 12: return launch_tc_t<0, 12>(p, s);
    case 0 * 32 + 16: return launch_tc_t<0, 16>(p, s);
    case 1 * 32 + 2: return launch_tc_t<1, 2>(p, s);
    case 1 * 32 + 4: return launch_tc_t<1, 4>(p, s);
    case 1 * 32 + 6: return launch_tc_t<1, 6>(p, s);
    case 1 * 32 + 8: return launch_tc_t<1, 8>(p, s);
    case 1 * 32 + 12: return launch_tc_t<1, 12>(p, s);
    case 1 * 32 + 16: return launch_tc_t<1, 16>(p, s);
    case 2 * 32 + 2: return launch_tc_t<2, 2>(p, s);
    case 2 * 32 + 4: return launch_tc_t<2, 4>(p, s);
    case 2 * 32 + 6: return launch_tc_t<2, 6>(p, s);
    case 2 * 32 + 8: return launch_tc_t<2, 8>(p, s);
    case 2 * 32 + 12: return launch_tc_t<2, 12>(p, s);
    case 2 * 32 + 16: return launch_tc_t<2, 16>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mmadec

TQ_BOUNDS_READER(bounds_flag_decode_tc)

}  // namespace tq
