// Internal declarations shared by the ABI layer (abi.cu) and the kernel files.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "tq.h"

namespace tq {

constexpr int kBlockTokens = TQ_BLOCK_TOKENS;
constexpr int kMaxG = 8;          // query heads per KV head
constexpr int kMaxLevels = 16;    // 2^b1 for b1 <= 4 (codebook build)

// Geometry of the packed cache, as plain values for kernels.
struct Geom {
  int B, Hkv, d, b1, m, vbits, group, W, dtype;
  bool hadamard;      // Pi = H diag(s) / sqrt(d): rotations on CUDA cores as a butterfly
  int64_t capacity;
  int64_t block_bytes, region_bytes, ring_k_off, ring_v_off;
  int64_t total_bytes;  // the cache buffer's extent (bounds-checked build)
  int f_idx, f_sign, f_rnorm, f_vcode, f_vmeta;        // bytes per token per field
  int o_idx, o_sign, o_rho, o_rnorm, o_vcode, o_vscale, o_vmin;  // field offsets in a block
};

Geom geom_of(const tq_cache* c);

// Bounds-checked build: each kernel file's flag (the code of its first failed
// check, 0 if none; -1 if it could not be read), read and cleared.  In the normal
// build these return 0.
int bounds_flag_quant();
int bounds_flag_decode();
int bounds_flag_decode_mma();
int bounds_flag_wide();
int bounds_flag_prefill();
int bounds_flag_prefill_tc();

// Record a thread-local error message (printf-style) and return `status`.
int set_error(int status, const char* fmt, ...);

// ---- setup (setup_kernels.cu) ----
cudaError_t launch_codebook(int d, int bits, float* cent, float* bnd, cudaStream_t s);
cudaError_t launch_projections_hadamard(int d, int m, uint64_t seed, float* Pi, float* S, float* T,
                                       cudaStream_t s);
cudaError_t launch_projections(int d, int m, uint64_t seed, float* Pi, float* S, float* T,
                               double* ws, cudaStream_t s);

// ---- quantisation / append (quant_kernels.cu) ----
struct QuantSrc {
  // Token i of (b, h) in this launch is absolute token t = t_first + i.
  // Cache mode: t < n_old reads ring slot t mod W, else chunk row t - n_old.
  const void* K;
  const void* V;
  int64_t n;          // tokens per (b, h) in this launch
  int64_t t_first;
  int64_t n_old;      // cache mode only
  int64_t n_new;      // cache mode only (rows of the chunk)
};
struct QuantDst {  // token-major arrays (standalone calls)
  uint8_t* idx;
  uint8_t* signs;
  float* rho;
  float* rnorm;
  uint8_t* codes;
  float* vscale;
  float* vmin;
};
// Read and clear the sticky flag the tensor-core quantise kernel raises when a
// bounded wait gives up (synchronises `s`).
cudaError_t quantize_error_flag(int* flag, cudaStream_t s);
cudaError_t launch_quantize_arrays(const QuantSrc& src, int dtype, int d, int b1, int m,
                                   int vbits, int group, bool do_keys, bool do_values,
                                   const float* Pi, const float* T, const float* cent,
                                   const float* bnd, const QuantDst& dst, cudaStream_t s);
// *ring_written (may be null): the launch also wrote the new ring (then no ring
// write may follow it)
cudaError_t launch_quantize_cache(const QuantSrc& src, const Geom& g, uint8_t* base,
                                  const float* Pi, const float* T, const float* cent,
                                  const float* bnd, cudaStream_t s, bool* ring_written);
cudaError_t launch_ring_write(const Geom& g, uint8_t* base, const void* K, const void* V,
                              int64_t n_old, int64_t n_new, cudaStream_t s);
// Decode step (tq_decode_step): quantise of the tokens leaving the ring with the
// ring write fused in, ring writes of incoming tokens into empty slots, and the
// tensor-core query preparation, in one launch.
struct DecodeWs;
cudaError_t launch_decode_step_pre(const QuantSrc& src, int64_t n_ring_only, const Geom& g,
                                   uint8_t* base, const float* Pi, const float* T,
                                   const float* cent, const float* bnd, const void* Q, int Hq,
                                   const float* S, float softmax_scale, const DecodeWs& ws,
                                   cudaStream_t s);

// ---- decode (decode_kernels.cu) ----
struct DecodeWs {
  float* qf;        // [B*Hq, d]   query in fp32
  float* qr;        // [B*Hq, d]   Pi q
  float* qs;        // [B*Hq, m]   sqrt(pi/2)/m * S q
  uint32_t* frag;   // [B*Hkv, ksteps, 2, 2, 32]  int8 query slices (tensor-core path)
  float* qconst;    // [B*Hkv, 8, 4]  per-head logit constants (tensor-core path)
  int* err;         // error flag set by a kernel whose bounded wait gave up
  int* counter;     // [B*Hkv] finished splits of each unit (fused combine)
  float* part_ml;   // [B*Hq, splits, 2]
  float* part_o;    // [B*Hq, splits, d]
};
size_t decode_ws_bytes(const Geom& g, int Hq, int splits);
// Scratch of a decode of c's current state with these arguments (abi.cu; 0 when
// they are invalid), and the device address of the static scratch array of
// tq_decode_attention_noalloc on the current device (noalloc_decode.cu).
size_t decode_ws_bytes_now(const tq_cache* c, int Hq, int num_splits);
int noalloc_scratch(void** out);
DecodeWs decode_ws_carve(void* base, const Geom& g, int Hq, int splits);
int decode_auto_splits(const Geom& g, int G, int64_t n_comp);
// The largest decode_auto_splits(g, G, n) for n <= capacity (workspace sizing).
int decode_max_auto_splits(const Geom& g, int G, int64_t capacity);

// tensor-core path (decode_mma.cu)
bool decode_mma_supported(const Geom& g, int G);
int decode_mma_ctas_per_sm(const Geom& g);      // resident CTAs per SM of the partial kernel
cudaError_t launch_decode_prep_mma(const Geom& g, const void* Q, int Hq, const float* Pi,
                                   const float* S, const float* cent, float scale,
                                   const DecodeWs& ws, cudaStream_t s);
// early_blk: packed blocks [0, early_blk) of every unit are not written by the kernel
// launched just before on the stream (0 when that is not known)
cudaError_t launch_decode_partial_mma(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                      float scale, float* logits, int splits, const DecodeWs& ws,
                                      void* out, int64_t early_blk, cudaStream_t s);

cudaError_t launch_decode_prep(const Geom& g, const void* Q, int Hq, const float* Pi,
                               const float* S, const DecodeWs& ws, cudaStream_t s);
cudaError_t launch_decode_partial(const Geom& g, const uint8_t* base, int64_t n_total,
                                  int Hq, float scale, const float* cent, float* logits,
                                  int splits, const DecodeWs& ws, cudaStream_t s, int qdiv = 1,
                                  int nslots = 0, bool with_ring = true);
cudaError_t launch_decode_combine(const Geom& g, int Hq, void* out, int splits,
                                  const DecodeWs& ws, cudaStream_t s);

// ---- multi-token (chunked prefill) attention (prefill_mma.cu) ----
// The chunk's n query tokens are a virtual batch of B * n decode queries; the
// history partials take slots 0..splits-1 of splits + 1, the exact segment (ring +
// chunk tokens 0..i) the last slot, and the decode combine merges them.
bool prefill_mma_supported(const Geom& g, int G);
// the tcgen05 history partial (prefill_tc.cu): chunks of >= 8 tokens on the
// tensor-core shapes whose operands fit
bool prefill_tc_supported(const Geom& g, int G, int nq);
int prefill_tc_splits(const Geom& g, int64_t n_comp, int nq);
cudaError_t launch_prefill_partial_tc(const Geom& g, const uint8_t* base, int64_t n_total, int Hq, int nq,
                                      int splits, int nslots, const float* cent, const DecodeWs& ws,
                                      cudaStream_t s);
int prefill_mma_warps(const Geom& g, int nq);
int prefill_auto_splits(const Geom& g, int G, int64_t n_comp, int nq, bool mma);
cudaError_t launch_prefill_partial_mma(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                       int nq, int splits, int nslots, const DecodeWs& ws,
                                       cudaStream_t s);
cudaError_t launch_prefill_exact(const Geom& g, const uint8_t* base, int64_t n_total, int Hq,
                                 int nq, const void* K, const void* V, float scale, int nslots,
                                 int slot, const DecodeWs& ws, cudaStream_t s);

// ---- sensitivity profile (sensitivity.cu) ----
size_t key_moments_ws_bytes();
cudaError_t launch_key_moments(const void* K, int dtype, int64_t n, double* out, double* part,
                               cudaStream_t s);
void sensitivity_segment(const double* var, int L, int k, int* bounds);
int sensitivity_allocate(const double* var, int L, const int* bounds, int k, int m_avg, int m_min,
                         int m_max, int* m);

// Launch with programmatic stream serialisation (programmatic dependent launch):
// the kernel may begin once the previous kernel of the stream has let its
// dependents launch (griddepcontrol.launch_dependents) instead of after that
// kernel completes.  Every kernel launched this way executes
// griddepcontrol.wait before it touches memory the previous kernel writes or
// reads, so stream order is kept for data, and completion still chains.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace tq
