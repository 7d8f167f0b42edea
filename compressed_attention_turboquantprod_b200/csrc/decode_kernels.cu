// Decode attention on the packed cache ([TQ] 四-六; [AQJL] QJL):
//   prep     per (b, query head): q in fp32, Pi q, sqrt(pi/2)/m S q  (rotate the
//            query forward and sketch it once, never the keys back)
//   partial  per (b, kv head, split): stream the split's 64-token blocks,
//            logits rho <Pi q, c[idx]> + ||r|| <qs, +-1> straight from the bits,
//            online softmax (base 2), P V with v = mn + code * s; the last split
//            also folds in the ring tokens exactly; writes (m, l, o) per head
//   combine  per (b, query head): merge the splits' (m, l, o).
#include <cfloat>

#include "common.cuh"

namespace tq {
namespace {

constexpr int DT = 256;           // threads of the partial kernel
constexpr int RC = 16;            // ring tokens per step
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTargetCtas = 148 * 4;

struct DParams {
  Geom g;
  const uint8_t* base;
  int64_t n_comp, n_total;
  int n_ring, Hq, G;
  float scale_log2;
  const float* cent;
  float* logits;
  int64_t n_log;
  int splits, bps;
  int qdiv;      // virtual batches per cache batch (query tokens of a chunk; 1 for a decode)
  int nslots;    // partial slots per (batch, query head); the split index is the slot
  DecodeWs ws;
};

__global__ void __launch_bounds__(DT) k_decode_partial(DParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const Geom& g = p.g;
  const int d = g.d, m = g.m, G = p.G, b1 = g.b1;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / g.Hkv, h = bh % g.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  float* sQr = reinterpret_cast<float*>(smem_raw);     // [G][d]
  float* sQs = sQr + G * d;                            // [G][m]
  float* sQf = sQs + G * m;                            // [G][d]
  float* sL = sQf + G * d;                             // [G][64]
  float* sP = sL + G * 64;                             // [G][64]
  float* sCent = sP + G * 64;                          // [16]
  float* sM = sCent + 16;                              // [G]
  float* sLs = sM + kMaxG;                             // [G]
  float* sAl = sLs + kMaxG;                            // [G]
  unsigned char* sBuf = reinterpret_cast<unsigned char*>(sAl + kMaxG);   // block / ring stage

  const int bq0 = b * p.Hq + h * G;
  for (int i = tid; i < G * d; i += DT) {
    sQr[i] = b1 > 0 ? p.ws.qr[(int64_t)bq0 * d + i] : 0.f;
    sQf[i] = p.ws.qf[(int64_t)bq0 * d + i];
  }
  for (int i = tid; i < G * m; i += DT) sQs[i] = p.ws.qs[(int64_t)bq0 * m + i];
  if (tid < 16) sCent[tid] = (b1 > 0 && tid < (1 << b1)) ? p.cent[tid] : 0.f;
  if (tid < kMaxG) {
    sM[tid] = -INFINITY;
    sLs[tid] = 0.f;
    sAl[tid] = 1.f;
  }
  __syncthreads();

  const int nhs = DT / d;                 // head sets in the P V mapping
  const int ch = tid % d, hs = tid / d;
  float acc[kMaxG];
#pragma unroll
  for (int k = 0; k < kMaxG; ++k) acc[k] = 0.f;

  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  const int64_t blk0 = (int64_t)split * p.bps;
  const int64_t blk1 = min(nblk, blk0 + p.bps);
  const uint8_t* region = p.base + (int64_t)((b / p.qdiv) * g.Hkv + h) * g.region_bytes;
  const int vmask = (1 << g.vbits) - 1;
  const int ng = d / g.group;

  auto softmax_step = [&]() {
    if (warp < G) {
      const int hh = warp;
      const float v0 = sL[hh * 64 + lane], v1 = sL[hh * 64 + lane + 32];
      const float mx = warp_max(fmaxf(v0, v1));
      const float m_old = sM[hh];
      const float m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {
        alpha = exp2f(m_old - m_new);
        p0 = exp2f(v0 - m_new);
        p1 = exp2f(v1 - m_new);
      }
      const float sum = warp_sum(p0 + p1);
      sP[hh * 64 + lane] = p0;
      sP[hh * 64 + lane + 32] = p1;
      if (lane == 0) {
        sLs[hh] = sLs[hh] * alpha + sum;
        sM[hh] = m_new;
        sAl[hh] = alpha;
      }
    }
  };

  for (int64_t blk = blk0; blk < blk1; ++blk) {
    {
      const uint4* src = reinterpret_cast<const uint4*>(region + blk * g.block_bytes);
      uint4* dst = reinterpret_cast<uint4*>(sBuf);
      const bool inb = TQ_CHECKED(src, g.block_bytes, p.base, g.total_bytes, 501);
      for (int i = tid; i < (int)(g.block_bytes / 16); i += DT)
        dst[i] = inb ? src[i] : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    const int nt = (int)min((int64_t)kBlockTokens, p.n_comp - blk * kBlockTokens);
    for (int pr = tid; pr < kBlockTokens * G; pr += DT) {
      const int tk = pr % kBlockTokens, hh = pr / kBlockTokens;
      float l2 = -INFINITY;
      if (tk < nt) {
        const float rho = reinterpret_cast<const float*>(sBuf + g.o_rho)[tk];
        float qjl = 0.f;
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(sBuf + g.o_sign + tk * g.f_sign);
        const float* qs = sQs + hh * m;
        for (int wi = 0; wi < m / 32; ++wi) {
          const uint32_t w = sw[wi];
#pragma unroll 8
          for (int ii = 0; ii < 32; ++ii) {
            const float q = qs[wi * 32 + ii];
            qjl += ((w >> ii) & 1u) ? q : -q;
          }
        }
        float logit;
        if (b1 > 0) {
          const float rn = reinterpret_cast<const float*>(sBuf + g.o_rnorm)[tk];
          const uint8_t* ib = sBuf + g.o_idx + tk * g.f_idx;
          const float* qr = sQr + hh * d;
          float mse = 0.f;
          for (int wi = 0; wi < d / 32; ++wi) {
            const uint32_t w0 = reinterpret_cast<const uint32_t*>(ib)[wi];
            const uint32_t w1 = b1 > 1 ? reinterpret_cast<const uint32_t*>(ib + d / 8)[wi] : 0u;
            const uint32_t w2 = b1 > 2 ? reinterpret_cast<const uint32_t*>(ib + d / 4)[wi] : 0u;
#pragma unroll 8
            for (int jj = 0; jj < 32; ++jj) {
              const int idx = ((w0 >> jj) & 1u) | (((w1 >> jj) & 1u) << 1) | (((w2 >> jj) & 1u) << 2);
              mse = fmaf(qr[wi * 32 + jj], sCent[idx], mse);
            }
          }
          logit = rho * mse + rn * qjl;
        } else {
          logit = rho * qjl;
        }
        if (p.logits) p.logits[(int64_t)(bq0 + hh) * p.n_log + blk * kBlockTokens + tk] = logit;
        l2 = logit * p.scale_log2;
      }
      sL[hh * 64 + tk] = l2;
    }
    __syncthreads();
    softmax_step();
    __syncthreads();
    {
      const float* vs = reinterpret_cast<const float*>(sBuf + g.o_vscale);
      const float* vm = reinterpret_cast<const float*>(sBuf + g.o_vmin);
      const int gi = ch / g.group;
      const int bit = ch * g.vbits;
      const int hoff = g.o_vcode + vcode_half_off(g, 0, bit >> 4);   // token-pair records
#pragma unroll
      for (int k = 0; k < kMaxG; ++k) {
        const int hh = hs + k * nhs;
        if (hh < G) acc[k] *= sAl[hh];
      }
      for (int tk = 0; tk < nt; ++tk) {
        const int code = (*reinterpret_cast<const uint16_t*>(sBuf + hoff + (tk >> 1) * 2 * g.f_vcode +
                                                              2 * (tk & 1)) >> (bit & 15)) & vmask;
        const float v = fmaf((float)code, vs[tk * ng + gi], vm[tk * ng + gi]);
#pragma unroll
        for (int k = 0; k < kMaxG; ++k) {
          const int hh = hs + k * nhs;
          if (hh < G) acc[k] = fmaf(sP[hh * 64 + tk], v, acc[k]);
        }
      }
    }
    __syncthreads();
  }

  if (split == p.splits - 1 && p.n_ring > 0) {
    const int es = (g.dtype == TQ_F32) ? 4 : 2;
    float* sK = reinterpret_cast<float*>(sBuf);     // [RC][d]
    float* sV = sK + RC * d;                        // [RC][d]
    const int64_t first = p.n_total - p.n_ring;
    for (int r0 = 0; r0 < p.n_ring; r0 += RC) {
      const int rows = min(RC, p.n_ring - r0);
      for (int i = tid; i < rows * d; i += DT) {
        const int rr = i / d, c = i % d;
        const int64_t slot = (first + r0 + rr) % g.W;
        const int64_t e = ((int64_t)bh * g.W + slot) * d + c;
        const bool inb = TQ_CHECKED(p.base + g.ring_v_off + e * es, es, p.base, g.total_bytes, 502);
        sK[rr * d + c] = inb ? load_f(p.base + g.ring_k_off, e, g.dtype) : 0.f;
        sV[rr * d + c] = inb ? load_f(p.base + g.ring_v_off, e, g.dtype) : 0.f;
      }
      (void)es;
      __syncthreads();
      for (int pr = tid; pr < kBlockTokens * G; pr += DT) {
        const int tk = pr % kBlockTokens, hh = pr / kBlockTokens;
        float l2 = -INFINITY;
        if (tk < rows) {
          float dot = 0.f;
          for (int j = 0; j < d; ++j) dot = fmaf(sQf[hh * d + j], sK[tk * d + j], dot);
          if (p.logits) p.logits[(int64_t)(bq0 + hh) * p.n_log + p.n_comp + r0 + tk] = dot;
          l2 = dot * p.scale_log2;
        }
        sL[hh * 64 + tk] = l2;
      }
      __syncthreads();
      softmax_step();
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kMaxG; ++k) {
        const int hh = hs + k * nhs;
        if (hh < G) acc[k] *= sAl[hh];
      }
      for (int tk = 0; tk < rows; ++tk) {
        const float v = sV[tk * d + ch];
#pragma unroll
        for (int k = 0; k < kMaxG; ++k) {
          const int hh = hs + k * nhs;
          if (hh < G) acc[k] = fmaf(sP[hh * 64 + tk], v, acc[k]);
        }
      }
      __syncthreads();
    }
  }

  for (int k = 0; k < kMaxG; ++k) {
    const int hh = hs + k * nhs;
    if (hh < G) p.ws.part_o[((int64_t)(bq0 + hh) * p.nslots + split) * d + ch] = acc[k];
  }
  if (tid < G) {
    p.ws.part_ml[((int64_t)(bq0 + tid) * p.nslots + split) * 2 + 0] = sM[tid];
    p.ws.part_ml[((int64_t)(bq0 + tid) * p.nslots + split) * 2 + 1] = sLs[tid];
  }
}

__global__ void __launch_bounds__(256) k_decode_prep(Geom g, const void* Q, int Hq, const float* Pi,
                                                     const float* S, DecodeWs ws) {
  __shared__ float sq[256];
  const int bq = blockIdx.x, d = g.d, m = g.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (bq == 0 && tid == 0) *ws.err = 0;
  for (int i = tid; i < d; i += blockDim.x) {
    const float v = load_f(Q, (int64_t)bq * d + i, g.dtype);
    sq[i] = v;
    ws.qf[(int64_t)bq * d + i] = v;
  }
  __syncthreads();
  const float qscale = 1.2533141373155003f / (float)m;   // sqrt(pi/2) / m
  const int rows_pi = (g.b1 > 0) ? d : 0;
  if (g.hadamard && warp == 0)      // Pi q as a butterfly: H (Pi[0,:] * q)
    warp_hadamard_rotate(Pi, sq, 1.f, ws.qr + (int64_t)bq * d, d, lane);
  for (int r = g.hadamard ? rows_pi + warp : warp; r < rows_pi + m; r += blockDim.x / 32) {
    const float* row = (r < rows_pi) ? Pi + (int64_t)r * d : S + (int64_t)(r - rows_pi) * d;
    float a = 0.f;
    for (int i = lane; i < d; i += 32) a = fmaf(row[i], sq[i], a);
    a = warp_sum(a);
    if (lane == 0) {
      if (r < rows_pi) ws.qr[(int64_t)bq * d + r] = a;
      else ws.qs[(int64_t)bq * m + (r - rows_pi)] = a * qscale;
    }
  }
}

__global__ void k_decode_combine(Geom g, int splits, void* out, DecodeWs ws) {
  const int bq = blockIdx.x, d = g.d;
  const float* ml = ws.part_ml + (int64_t)bq * splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ml[2 * s]);
  const float* po = ws.part_o + (int64_t)bq * splits * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
      // the same sums in the same order; four splits' values are loaded before
      // any is used, so that their loads are in flight together
      int s = 0;
      for (; s + 4 <= splits; s += 4) {
        float v[4], ms[4], ls[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          ms[u] = ml[2 * (s + u)];
          ls[u] = ml[2 * (s + u) + 1];
          v[u] = po[(int64_t)(s + u) * d + c];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (ms[u] != -INFINITY) {
            const float w = exp2f(ms[u] - M);
            L = fmaf(ls[u], w, L);
            o = fmaf(v[u], w, o);
          }
      }
      for (; s < splits; ++s) {
        const float m1 = ml[2 * s];
        if (m1 == -INFINITY) continue;
        const float w = exp2f(m1 - M);
        L = fmaf(ml[2 * s + 1], w, L);
        o = fmaf(po[(int64_t)s * d + c], w, o);
      }
      o = o / L;
    }
    store_f(out, (int64_t)bq * d + c, g.dtype, o);
  }
}

size_t partial_smem(const Geom& g, int G) {
  const size_t q = sizeof(float) * ((size_t)G * (2 * g.d + g.m) + 2 * G * 64 + 16 + 3 * kMaxG);
  const size_t ring = sizeof(float) * 2 * RC * g.d;
  const size_t stage = (size_t)g.block_bytes > ring ? (size_t)g.block_bytes : ring;
  return ((q + 15) / 16) * 16 + stage;
}

}  // namespace

static inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static size_t frag_words(const Geom& g) {
  const int F = g.b1 > 0 ? 1 << (g.b1 - 1) : 0;
  return (size_t)(F * g.d / 32 + g.m / 32) * 2 * 2 * 32;
}

size_t decode_ws_bytes(const Geom& g, int Hq, int splits) {
  const size_t bq = (size_t)g.B * Hq, units = (size_t)g.B * g.Hkv;
  size_t o = 0;
  o += align256(bq * g.d * sizeof(float));                // qf
  o += align256(bq * g.d * sizeof(float));                // qr
  o += align256(bq * g.m * sizeof(float));                // qs
  o += align256(units * frag_words(g) * sizeof(uint32_t)); // frag
  o += align256(units * 8 * 4 * sizeof(float));           // qconst
  o += 256;                                               // err
  o += align256(units * sizeof(int));                     // counter
  o += align256(bq * splits * 2 * sizeof(float));         // part_ml
  o += align256(bq * splits * g.d * sizeof(float));       // part_o
  return o;
}

DecodeWs decode_ws_carve(void* base, const Geom& g, int Hq, int splits) {
  const size_t bq = (size_t)g.B * Hq, units = (size_t)g.B * g.Hkv;
  char* p = static_cast<char*>(base);
  DecodeWs w;
  w.qf = reinterpret_cast<float*>(p);
  p += align256(bq * g.d * sizeof(float));
  w.qr = reinterpret_cast<float*>(p);
  p += align256(bq * g.d * sizeof(float));
  w.qs = reinterpret_cast<float*>(p);
  p += align256(bq * g.m * sizeof(float));
  w.frag = reinterpret_cast<uint32_t*>(p);
  p += align256(units * frag_words(g) * sizeof(uint32_t));
  w.qconst = reinterpret_cast<float*>(p);
  p += align256(units * 8 * 4 * sizeof(float));
  w.err = reinterpret_cast<int*>(p);
  p += 256;
  w.counter = reinterpret_cast<int*>(p);
  p += align256(units * sizeof(int));
  w.part_ml = reinterpret_cast<float*>(p);
  p += align256(bq * splits * 2 * sizeof(float));
  w.part_o = reinterpret_cast<float*>(p);
  return w;
}

// The tensor-core kernel's CTAs of a unit split its blocks evenly; the SM that ends
// last carries about ceil(units s / 148) CTAs of ceil(nblk / s) blocks (CTAs that
// finish early are backfilled by waiting ones), the per-SM load this returns.
static int64_t sm_load(int64_t units, int64_t s, int64_t nblk) {
  return ((units * s + 147) / 148) * ((nblk + s - 1) / s);
}

int decode_auto_splits(const Geom& g, int G, int64_t n_comp) {
  const int64_t nblk = (n_comp + kBlockTokens - 1) / kBlockTokens;
  const int units = g.B * g.Hkv;
  int64_t s;
  if (decode_mma_supported(g, G)) {
    // one wave of the kernel (148 SMs x its resident CTAs); twice that many smaller
    // CTAs when the wave leaves the SMs' loads uneven (e.g. 128 units x 4 splits in
    // 592 slots: 4 CTAs on some SMs, 3 on others) and the halves balance them at
    // least 5 % better
    const int64_t s1 = (int64_t)(148 * decode_mma_ctas_per_sm(g)) / units;
    s = s1;
    if (s1 >= 1 && 2 * s1 <= nblk && sm_load(units, 2 * s1, nblk) * 20 < sm_load(units, s1, nblk) * 19)
      s = 2 * s1;
  } else {
    s = (kTargetCtas + units - 1) / units;
  }
  if (s > nblk) s = nblk;
  if (s < 1) s = 1;
  return (int)s;
}

int decode_max_auto_splits(const Geom& g, int G, int64_t capacity) {
  if (!decode_mma_supported(g, G)) return decode_auto_splits(g, G, capacity);   // grows with n
  const int64_t nblk = (capacity + kBlockTokens - 1) / kBlockTokens;
  int64_t s = 2 * ((int64_t)(148 * decode_mma_ctas_per_sm(g)) / (g.B * g.Hkv));
  if (s > nblk) s = nblk;
  return s < 1 ? 1 : (int)s;
}

cudaError_t launch_decode_prep(const Geom& g, const void* Q, int Hq, const float* Pi,
                               const float* S, const DecodeWs& ws, cudaStream_t s) {
  k_decode_prep<<<g.B * Hq, 256, 0, s>>>(g, Q, Hq, Pi, S, ws);
  return cudaGetLastError();
}

cudaError_t launch_decode_partial(const Geom& g, const uint8_t* base, int64_t n_total,
                                  int Hq, float scale, const float* cent, float* logits,
                                  int splits, const DecodeWs& ws, cudaStream_t s, int qdiv,
                                  int nslots, bool with_ring) {
  DParams p{};
  p.g = g;
  p.base = base;
  p.n_total = n_total;
  p.n_comp = n_total > g.W ? n_total - g.W : 0;
  p.n_ring = with_ring ? (int)(n_total < g.W ? n_total : g.W) : 0;
  p.qdiv = qdiv;
  p.nslots = nslots > 0 ? nslots : splits;
  p.Hq = Hq;
  p.G = Hq / g.Hkv;
  p.scale_log2 = scale * kLog2e;
  p.cent = cent;
  p.logits = logits;
  p.n_log = p.n_comp + p.n_ring;
  const int64_t nblk = (p.n_comp + kBlockTokens - 1) / kBlockTokens;
  p.splits = splits;
  p.bps = (int)((nblk + splits - 1) / splits);
  p.ws = ws;
  const size_t smem = partial_smem(g, p.G);
  cudaError_t e = cudaFuncSetAttribute(k_decode_partial,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)splits, (unsigned)(g.B * g.Hkv));
  k_decode_partial<<<grid, DT, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const Geom& g, int Hq, void* out, int splits,
                                  const DecodeWs& ws, cudaStream_t s) {
  k_decode_combine<<<g.B * Hq, g.d, 0, s>>>(g, splits, out, ws);
  return cudaGetLastError();
}

TQ_BOUNDS_READER(bounds_flag_decode)

}  // namespace tq
