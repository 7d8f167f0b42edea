// C ABI of libtq: argument checks, cache layout, dispatch to the kernels.
// Every check runs on the host before any launch; a failed check launches
// nothing and writes nothing.
#include <cctype>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "tq_internal.h"

namespace {

thread_local std::string g_err;
std::mutex g_fault_mu;
std::string g_fault;
bool g_fault_env_read = false;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return status;
}

int ok() {
  g_err.clear();
  return TQ_OK;
}

// Host-side fault injection: returns true (and clears it) if `name` is armed.
bool injected(const char* name) {
  std::lock_guard<std::mutex> lk(g_fault_mu);
  if (!g_fault_env_read) {
    g_fault_env_read = true;
    const char* e = std::getenv("TQ_FAULT");
    if (e && *e) g_fault = e;
  }
  if (!g_fault.empty() && g_fault == name) {
    g_fault.clear();
    return true;
  }
  return false;
}

#define TQ_FAULT_POINT(name)                                          \
  do {                                                                \
    if (injected(name)) return fail(TQ_ERR_CUDA, "injected fault");   \
  } while (0)

int cuda_fail(cudaError_t e, const char* where) {
  return fail(TQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// A CUDA error left pending by earlier asynchronous work.
int check_pending(const char* where) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, where);
  return TQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(int dt) { return dt == TQ_F32 || dt == TQ_F16 || dt == TQ_BF16; }
bool valid_d(int d) { return d == 64 || d == 128 || d == 256; }
bool valid_m(int m) { return m >= 32 && m <= 1024 && m % 32 == 0; }
bool valid_group(int g, int d) {
  return (g == 16 || g == 32 || g == 64 || g == 128) && g <= d && d % g == 0;
}
size_t esize(int dt) { return dt == TQ_F32 ? 4 : 2; }
size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int check_shape(int d, int b1, int m, int vbits, int group, bool need_values) {
  if (!valid_d(d)) return fail(TQ_ERR_UNSUPPORTED, "head dim d=%d not in {64,128,256}", d);
  if (b1 < 0 || b1 > 3) return fail(TQ_ERR_UNSUPPORTED, "b1=%d not in [0,3]", b1);
  if (!valid_m(m)) return fail(TQ_ERR_UNSUPPORTED, "sketch dim m=%d not a multiple of 32 in [32,1024]", m);
  if (need_values) {
    if (vbits != 2 && vbits != 4) return fail(TQ_ERR_UNSUPPORTED, "vbits=%d not in {2,4}", vbits);
    if (!valid_group(group, d)) return fail(TQ_ERR_UNSUPPORTED, "value group %d invalid for d=%d", group, d);
  }
  return TQ_OK;
}

// Cache layout from a descriptor: status, and the layout in *out (may be null).
int layout_status(const tq_cache_desc* dsc, tq_cache* out) {
  if (!dsc) return fail(TQ_ERR_INVALID_ARG, "null descriptor");
  if (dsc->B < 1 || dsc->Hkv < 1 || dsc->capacity < 0 || dsc->W < 0 || dsc->W > 1024)
    return fail(TQ_ERR_INVALID_ARG, "bad descriptor (B=%d Hkv=%d capacity=%lld W=%d)", dsc->B,
                dsc->Hkv, (long long)dsc->capacity, dsc->W);
  if (!valid_dtype(dsc->dtype)) return fail(TQ_ERR_INVALID_ARG, "bad dtype %d", dsc->dtype);
  if (dsc->rotation != TQ_ROTATION_DENSE && dsc->rotation != TQ_ROTATION_HADAMARD)
    return fail(TQ_ERR_INVALID_ARG, "bad rotation %d", dsc->rotation);
  int st = check_shape(dsc->d, dsc->b1, dsc->m, dsc->vbits, dsc->group, true);
  if (st != TQ_OK) return st;
  const int d = dsc->d, b1 = dsc->b1;
  const int f_idx = b1 * d / 8, f_sign = dsc->m / 8, f_rnorm = b1 > 0 ? 4 : 0;
  const int f_vcode = d * dsc->vbits / 8, f_vmeta = 4 * (d / dsc->group);
  const int T = tq::kBlockTokens;
  tq_cache c;
  std::memset(&c, 0, sizeof(c));
  c.desc = *dsc;
  int64_t o = 0;
  c.o_idx = (int32_t)o;    o += (int64_t)T * f_idx;
  c.o_sign = (int32_t)o;   o += (int64_t)T * f_sign;
  c.o_rho = (int32_t)o;    o += (int64_t)T * 4;
  c.o_rnorm = (int32_t)o;  o += (int64_t)T * f_rnorm;
  c.o_vcode = (int32_t)o;  o += (int64_t)T * f_vcode;
  c.o_vscale = (int32_t)o; o += (int64_t)T * f_vmeta;
  c.o_vmin = (int32_t)o;   o += (int64_t)T * f_vmeta;
  c.block_bytes = o;
  c.token_bytes = f_idx + f_sign + 4 + f_rnorm + f_vcode + 2 * f_vmeta;
  const int64_t nblk = (dsc->capacity + T - 1) / T;
  c.region_bytes = nblk * c.block_bytes;
  const size_t packed = (size_t)dsc->B * dsc->Hkv * (size_t)c.region_bytes;
  const size_t ring = (size_t)dsc->B * dsc->Hkv * dsc->W * d * esize(dsc->dtype);
  c.ring_k_off = (int64_t)align256(packed);
  c.ring_v_off = (int64_t)align256((size_t)c.ring_k_off + ring);
  const size_t total = align256((size_t)c.ring_v_off + ring);
  c.bytes = total;
  if (out) *out = c;
  return TQ_OK;
}

// Total bytes of the layout, 0 if the descriptor is invalid.
size_t layout(const tq_cache_desc* dsc, tq_cache* out) {
  tq_cache c;
  if (layout_status(dsc, &c) != TQ_OK) return 0;
  if (out) *out = c;
  return c.bytes;
}

int64_t n_comp_of(const tq_cache* c) {
  return c->n_total > c->desc.W ? c->n_total - c->desc.W : 0;
}

int check_cache(const tq_cache* c) {
  if (!c || !c->base) return fail(TQ_ERR_INVALID_ARG, "null cache or cache without memory");
  tq_cache ref;
  int lst = layout_status(&c->desc, &ref);
  if (lst != TQ_OK) return lst;
  if (ref.block_bytes != c->block_bytes || ref.ring_k_off != c->ring_k_off || c->bytes < ref.bytes)
    return fail(TQ_ERR_INVALID_ARG, "cache struct does not match its descriptor (not initialised?)");
  if (c->n_total < 0) return fail(TQ_ERR_INVALID_ARG, "negative token count");
  return TQ_OK;
}

// Effective split count and the partition it implies.
int eff_splits(const tq::Geom& g, int G, int64_t n_comp, int num_splits) {
  const int64_t nblk = (n_comp + tq::kBlockTokens - 1) / tq::kBlockTokens;
  int s = num_splits > 0 ? num_splits : tq::decode_auto_splits(g, G, n_comp);
  if (nblk == 0) return 1;
  if (s > nblk) s = (int)nblk;
  const int64_t bps = (nblk + s - 1) / s;
  return (int)((nblk + bps - 1) / bps);
}

int max_splits(const tq_cache* c, int Hq, int num_splits) {
  if (num_splits > 0) return num_splits;
  tq::Geom g = tq::geom_of(c);
  return tq::decode_max_auto_splits(g, Hq / c->desc.Hkv, c->desc.capacity);
}

int check_decode_common(const tq_cache* c, int Hq, int num_splits) {
  int st = check_cache(c);
  if (st != TQ_OK) return st;
  if (Hq < c->desc.Hkv || Hq % c->desc.Hkv != 0 || Hq / c->desc.Hkv > tq::kMaxG)
    return fail(TQ_ERR_UNSUPPORTED, "Hq=%d must be a multiple of Hkv=%d with at most %d heads per KV head",
                Hq, c->desc.Hkv, tq::kMaxG);
  if (num_splits < 0 || num_splits > 65535) return fail(TQ_ERR_INVALID_ARG, "num_splits=%d", num_splits);
  return TQ_OK;
}

}  // namespace

namespace tq {
int set_error(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return status;
}

Geom geom_of(const tq_cache* c) {
  Geom g;
  const tq_cache_desc& d = c->desc;
  g.B = d.B;
  g.Hkv = d.Hkv;
  g.d = d.d;
  g.b1 = d.b1;
  g.m = d.m;
  g.vbits = d.vbits;
  g.group = d.group;
  g.W = d.W;
  g.dtype = d.dtype;
  g.hadamard = d.rotation == TQ_ROTATION_HADAMARD && d.b1 > 0;
  g.capacity = d.capacity;
  g.block_bytes = c->block_bytes;
  g.region_bytes = c->region_bytes;
  g.ring_k_off = c->ring_k_off;
  g.ring_v_off = c->ring_v_off;
  g.total_bytes = (int64_t)c->bytes;
  g.f_idx = d.b1 * d.d / 8;
  g.f_sign = d.m / 8;
  g.f_rnorm = d.b1 > 0 ? 4 : 0;
  g.f_vcode = d.d * d.vbits / 8;
  g.f_vmeta = 4 * (d.d / d.group);
  g.o_idx = c->o_idx;
  g.o_sign = c->o_sign;
  g.o_rho = c->o_rho;
  g.o_rnorm = c->o_rnorm;
  g.o_vcode = c->o_vcode;
  g.o_vscale = c->o_vscale;
  g.o_vmin = c->o_vmin;
  return g;
}
}  // namespace tq

namespace tq {
// Scratch bytes a decode of the cache's current state needs: the split count is
// the one decode_plan takes (clamped to the cache's blocks), 0 for invalid
// arguments.
size_t decode_ws_bytes_now(const tq_cache* c, int Hq, int num_splits) {
  if (check_decode_common(c, Hq, num_splits) != TQ_OK) return 0;
  const Geom g = geom_of(c);
  return decode_ws_bytes(g, Hq, eff_splits(g, Hq / c->desc.Hkv, n_comp_of(c), num_splits));
}
}  // namespace tq

extern "C" {

const char* tq_last_error(void) { return g_err.c_str(); }

int tq_debug_bounds_enabled(void) {
#ifdef TQ_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

int tq_debug_bounds_check(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "tq_debug_bounds_check");
  const struct {
    const char* file;
    int (*read)();
  } files[] = {{"quant_kernels", tq::bounds_flag_quant}, {"decode_kernels", tq::bounds_flag_decode},
               {"decode_mma", tq::bounds_flag_decode_mma}, {"decode_mma_wide", tq::bounds_flag_wide},
               {"prefill_mma", tq::bounds_flag_prefill}, {"prefill_tc", tq::bounds_flag_prefill_tc}};
  int first = 0;
  const char* where = "";
  for (const auto& f : files) {
    const int v = f.read();
    if (v != 0 && first == 0) {
      first = v;
      where = f.file;
    }
  }
  if (first == -1) return fail(TQ_ERR_CUDA, "tq_debug_bounds_check: a flag could not be read");
  if (first != 0)
    return fail(TQ_ERR_CUDA, "bounds check %d failed in %s (an access outside its buffer was skipped)",
                first, where);
  return ok();
}

int tq_version(void) { return 1; }

int tq_debug_fail_next(const char* name) {
  std::lock_guard<std::mutex> lk(g_fault_mu);
  g_fault_env_read = true;
  g_fault = name ? name : "";
  return TQ_OK;
}

int tq_codebook_build(int d, int bits, float* centroids, float* boundaries, void* stream) {
  TQ_FAULT_POINT("tq_codebook_build");
  if (!centroids || !boundaries || !aligned16(centroids) || !aligned16(boundaries))
    return fail(TQ_ERR_INVALID_ARG, "centroids/boundaries must be non-null, 16-byte aligned");
  if (d < 16 || d > 4096) return fail(TQ_ERR_INVALID_ARG, "d=%d not in [16,4096]", d);
  if (bits < 1 || bits > 4) return fail(TQ_ERR_UNSUPPORTED, "bits=%d not in [1,4]", bits);
  int st = check_pending("tq_codebook_build");
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // A run that does not converge leaves centroids[0] = NaN; read it back.
  cudaError_t e = tq::launch_codebook(d, bits, centroids, boundaries, s);
  float c0 = 0.f;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&c0, centroids, sizeof(float), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_codebook_build");
  if (c0 != c0) return fail(TQ_ERR_NOT_CONVERGED, "Lloyd-Max iteration did not converge (d=%d bits=%d)", d, bits);
  return ok();
}

size_t tq_projections_workspace_bytes(int d) {
  if (d <= 0 || d > 256) return 0;
  return 2 * (size_t)d * d * sizeof(double);
}

int tq_make_projections_hadamard(int d, int m, int layer, uint64_t base_seed, uint64_t stride,
                                 float* Pi, float* S, float* T, void* stream) {
  TQ_FAULT_POINT("tq_make_projections_hadamard");
  if (!valid_d(d)) return fail(TQ_ERR_UNSUPPORTED, "head dim d=%d not in {64,128,256}", d);
  if (!valid_m(m)) return fail(TQ_ERR_UNSUPPORTED, "sketch dim m=%d not a multiple of 32 in [32,1024]", m);
  if (layer < 0) return fail(TQ_ERR_INVALID_ARG, "layer=%d", layer);
  if (!Pi || !S || !aligned16(Pi) || !aligned16(S) || (T && !aligned16(T)))
    return fail(TQ_ERR_INVALID_ARG, "Pi and S must be non-null; Pi, S, T 16-byte aligned");
  int st = check_pending("tq_make_projections_hadamard");
  if (st != TQ_OK) return st;
  const uint64_t seed = base_seed + stride * (uint64_t)layer;
  cudaError_t e = tq::launch_projections_hadamard(d, m, seed, Pi, S, T, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_make_projections_hadamard");
  return ok();
}

int tq_make_projections(int d, int m, int layer, uint64_t base_seed, uint64_t stride, float* Pi,
                        float* S, float* T, void* workspace, size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_make_projections");
  if (!valid_d(d)) return fail(TQ_ERR_UNSUPPORTED, "head dim d=%d not in {64,128,256}", d);
  if (!valid_m(m)) return fail(TQ_ERR_UNSUPPORTED, "sketch dim m=%d not a multiple of 32 in [32,1024]", m);
  if (layer < 0) return fail(TQ_ERR_INVALID_ARG, "layer=%d", layer);
  if (!S || !aligned16(S) || (Pi && !aligned16(Pi)) || (T && !aligned16(T)))
    return fail(TQ_ERR_INVALID_ARG, "S must be non-null; Pi, S, T 16-byte aligned");
  if (Pi && (!workspace || !aligned16(workspace) || ws_bytes < tq_projections_workspace_bytes(d)))
    return fail(TQ_ERR_INVALID_ARG, "workspace of %zu bytes needed", tq_projections_workspace_bytes(d));
  int st = check_pending("tq_make_projections");
  if (st != TQ_OK) return st;
  const uint64_t seed = base_seed + stride * (uint64_t)layer;
  cudaError_t e = tq::launch_projections(d, m, seed, Pi, S, T, static_cast<double*>(workspace),
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_make_projections");
  return ok();
}

int tq_quantize_keys(const void* K, int dtype, int64_t n, int d, int b1, int m, const float* Pi,
                     const float* T, const float* centroids, const float* boundaries,
                     uint8_t* idx_planes, uint8_t* signs, float* norm_x, float* norm_r,
                     void* stream) {
  TQ_FAULT_POINT("tq_quantize_keys");
  if (!valid_dtype(dtype)) return fail(TQ_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n=%lld", (long long)n);
  int st = check_shape(d, b1, m, 2, 32, false);
  if (st != TQ_OK) return st;
  if (!K || !T || !signs || !norm_x || !aligned16(K) || !aligned16(T) || !aligned16(signs))
    return fail(TQ_ERR_INVALID_ARG, "K, T, signs, norm_x must be non-null (K, T, signs 16-byte aligned)");
  if (b1 > 0 && (!Pi || !centroids || !boundaries || !idx_planes || !norm_r || !aligned16(Pi) ||
                 !aligned16(idx_planes)))
    return fail(TQ_ERR_INVALID_ARG, "b1>0 needs Pi, centroids, boundaries, idx_planes, norm_r");
  if (n == 0) return ok();
  st = check_pending("tq_quantize_keys");
  if (st != TQ_OK) return st;
  tq::QuantSrc src{K, nullptr, n, 0, 0, 0};
  tq::QuantDst dst{idx_planes, signs, norm_x, norm_r, nullptr, nullptr, nullptr};
  cudaError_t e = tq::launch_quantize_arrays(src, dtype, d, b1, m, 2, 32, true, false, Pi, T,
                                             centroids, boundaries, dst,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_quantize_keys");
  return ok();
}

int tq_quantize_values(const void* V, int dtype, int64_t n, int d, int vbits, int group,
                       uint8_t* codes, float* scale, float* vmin, void* stream) {
  TQ_FAULT_POINT("tq_quantize_values");
  if (!valid_dtype(dtype)) return fail(TQ_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n=%lld", (long long)n);
  int st = check_shape(d, 0, 32, vbits, group, true);
  if (st != TQ_OK) return st;
  if (!V || !codes || !scale || !vmin || !aligned16(V) || !aligned16(codes))
    return fail(TQ_ERR_INVALID_ARG, "V, codes, scale, vmin must be non-null (V, codes 16-byte aligned)");
  if (n == 0) return ok();
  st = check_pending("tq_quantize_values");
  if (st != TQ_OK) return st;
  tq::QuantSrc src{nullptr, V, n, 0, 0, 0};
  tq::QuantDst dst{nullptr, nullptr, nullptr, nullptr, codes, scale, vmin};
  cudaError_t e = tq::launch_quantize_arrays(src, dtype, d, 0, 32, vbits, group, false, true,
                                             nullptr, nullptr, nullptr, nullptr, dst,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_quantize_values");
  return ok();
}

size_t tq_cache_bytes(const tq_cache_desc* desc) { return layout(desc, nullptr); }

int tq_cache_layout(const tq_cache_desc* desc, tq_cache* out) {
  if (!out) return fail(TQ_ERR_INVALID_ARG, "null output");
  tq_cache c;
  int st = layout_status(desc, &c);
  if (st != TQ_OK) return st;
  *out = c;
  return ok();
}

int tq_cache_init(tq_cache* c, const tq_cache_desc* desc, void* dev_mem, size_t bytes,
                  void* stream) {
  TQ_FAULT_POINT("tq_cache_init");
  if (!c) return fail(TQ_ERR_INVALID_ARG, "null cache");
  tq_cache tmp;
  int lst = layout_status(desc, &tmp);
  if (lst != TQ_OK) return lst;
  const size_t need = tmp.bytes;
  if (!dev_mem || (reinterpret_cast<uintptr_t>(dev_mem) & 255u) != 0)
    return fail(TQ_ERR_INVALID_ARG, "cache memory must be non-null and 256-byte aligned");
  if (bytes < need) return fail(TQ_ERR_INVALID_ARG, "cache memory %zu bytes < %zu needed", bytes, need);
  int st = check_pending("tq_cache_init");
  if (st != TQ_OK) return st;
  cudaError_t e = cudaMemsetAsync(dev_mem, 0, need, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_cache_init");
  tmp.base = dev_mem;
  tmp.bytes = bytes;
  tmp.n_total = 0;
  *c = tmp;
  return ok();
}

int64_t tq_cache_compressed_tokens(const tq_cache* c) { return c ? n_comp_of(c) : 0; }
int64_t tq_cache_ring_tokens(const tq_cache* c) {
  if (!c) return 0;
  return c->n_total < c->desc.W ? c->n_total : c->desc.W;
}

// Arguments of an append of n_new >= 1 tokens; the compressed-token counts before
// and after go to *c_old / *c_new.
static int append_checks(const tq_cache* c, const void* K, const void* V, int64_t n_new,
                         const float* Pi, const float* T, const float* centroids,
                         const float* boundaries, int64_t* c_old_out, int64_t* c_new_out) {
  if (!K || !V || !aligned16(K) || !aligned16(V))
    return fail(TQ_ERR_INVALID_ARG, "K and V must be non-null and 16-byte aligned");
  const tq_cache_desc& dsc = c->desc;
  const int64_t n_old = c->n_total, n_tot = n_old + n_new;
  const int64_t c_old = n_old > dsc.W ? n_old - dsc.W : 0;
  const int64_t c_new = n_tot > dsc.W ? n_tot - dsc.W : 0;
  if (c_new > dsc.capacity)
    return fail(TQ_ERR_CAPACITY, "append of %lld tokens needs %lld compressed slots > capacity %lld",
                (long long)n_new, (long long)c_new, (long long)dsc.capacity);
  if (c_new > c_old) {
    if (!T || !aligned16(T) || (dsc.b1 > 0 && (!Pi || !centroids || !boundaries || !aligned16(Pi))))
      return fail(TQ_ERR_INVALID_ARG, "projections / codebook pointers missing");
  }
  *c_old_out = c_old;
  *c_new_out = c_new;
  return TQ_OK;
}

int tq_append(tq_cache* c, const void* K, const void* V, int64_t n_new, const float* Pi,
              const float* T, const float* centroids, const float* boundaries, void* stream) {
  TQ_FAULT_POINT("tq_append");
  int st = check_cache(c);
  if (st != TQ_OK) return st;
  if (n_new < 0) return fail(TQ_ERR_INVALID_ARG, "n_new=%lld", (long long)n_new);
  if (n_new == 0) return ok();
  const tq_cache_desc& dsc = c->desc;
  const int64_t n_old = c->n_total, n_tot = n_old + n_new;
  int64_t c_old = 0, c_new = 0;
  st = append_checks(c, K, V, n_new, Pi, T, centroids, boundaries, &c_old, &c_new);
  if (st != TQ_OK) return st;
  (void)dsc;
  st = check_pending("tq_append");
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  tq::Geom g = tq::geom_of(c);
  uint8_t* base = static_cast<uint8_t*>(c->base);
  cudaError_t e = cudaSuccess;
  bool ring_written = false;
  if (c_new > c_old) {
    tq::QuantSrc src{K, V, c_new - c_old, c_old, n_old, n_new};
    e = tq::launch_quantize_cache(src, g, base, Pi, T, centroids, boundaries, s, &ring_written);
    if (e != cudaSuccess) return cuda_fail(e, "tq_append: quantize");
  }
  if (!ring_written) {
    e = tq::launch_ring_write(g, base, K, V, n_old, n_new, s);
    if (e != cudaSuccess) return cuda_fail(e, "tq_append: ring");
  }
  c->n_total = n_tot;
  return ok();
}

int tq_decode_auto_splits(const tq_cache* c, int Hq) {
  if (check_decode_common(c, Hq, 0) != TQ_OK) return -1;
  return eff_splits(tq::geom_of(c), Hq / c->desc.Hkv, n_comp_of(c), 0);
}

size_t tq_decode_workspace_bytes(const tq_cache* c, int Hq, int num_splits) {
  if (check_decode_common(c, Hq, num_splits) != TQ_OK) return 0;
  return tq::decode_ws_bytes(tq::geom_of(c), Hq, max_splits(c, Hq, num_splits));
}


struct DecodePlan {
  tq::Geom g;
  int splits = 1;
  bool mma = false;
  tq::DecodeWs ws{};
};

// Every check of a decode (or of its stages) on cache state c, before any launch.
static int decode_plan(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                       const float* Pi, const float* S, const float* centroids, void* out,
                       int num_splits, void* workspace, size_t ws_bytes, bool prep, bool partial,
                       bool combine, const char* name, DecodePlan& P) {
  int st = check_decode_common(c, Hq, num_splits);
  if (st != TQ_OK) return st;
  const tq_cache_desc& dsc = c->desc;
  P.g = tq::geom_of(c);
  const int64_t n_comp = n_comp_of(c);
  const int G = Hq / dsc.Hkv;
  P.splits = eff_splits(P.g, G, n_comp, num_splits);
  P.mma = tq::decode_mma_supported(P.g, G);
  const size_t need = tq::decode_ws_bytes(P.g, Hq, P.splits);
  if (!workspace || !aligned16(workspace) || ws_bytes < need)
    return fail(TQ_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed", name, need);
  if (prep) {
    if (!Q || !S || !aligned16(S) || (dsc.b1 > 0 && (!Pi || !aligned16(Pi))))
      return fail(TQ_ERR_INVALID_ARG, "%s: Q, S (and Pi when b1>0) needed", name);
  }
  if (prep || partial) {
    if (!std::isfinite(softmax_scale)) return fail(TQ_ERR_INVALID_ARG, "%s: softmax_scale", name);
    if (dsc.b1 > 0 && !centroids) return fail(TQ_ERR_INVALID_ARG, "%s: centroids needed", name);
  }
  if (combine && !out) return fail(TQ_ERR_INVALID_ARG, "%s: out needed", name);
  P.ws = tq::decode_ws_carve(workspace, P.g, Hq, P.splits);
  return TQ_OK;
}

// early_blk: packed blocks [0, early_blk) of every unit that the kernel launched just
// before the partial kernel does not write (the partial may request them before it
// waits for that kernel); the preparation launched here writes none of them.
static int decode_launch(const tq_cache* c, const DecodePlan& P, const void* Q, int Hq,
                         float softmax_scale, const float* Pi, const float* S,
                         const float* centroids, void* out, float* logits, cudaStream_t s,
                         bool prep, bool partial, bool combine, const char* name,
                         int64_t early_blk = 0) {
  cudaError_t e = cudaSuccess;
  if (prep) {
    e = P.mma ? tq::launch_decode_prep_mma(P.g, Q, Hq, Pi, S, centroids, softmax_scale, P.ws, s)
              : tq::launch_decode_prep(P.g, Q, Hq, Pi, S, P.ws, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
  }
  if (partial) {
    // the tensor-core partial kernel merges the splits itself when given `out`
    void* fused_out = (P.mma && combine) ? out : nullptr;
    e = P.mma ? tq::launch_decode_partial_mma(P.g, static_cast<const uint8_t*>(c->base), c->n_total,
                                              Hq, softmax_scale, logits, P.splits, P.ws, fused_out,
                                              prep ? INT64_MAX : early_blk, s)
              : tq::launch_decode_partial(P.g, static_cast<const uint8_t*>(c->base), c->n_total, Hq,
                                          softmax_scale, centroids, logits, P.splits, P.ws, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    if (fused_out) combine = false;
  }
  if (combine) {
    e = tq::launch_decode_combine(P.g, Hq, out, P.splits, P.ws, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
  }
  return ok();
}

static int decode_stage(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                        const float* Pi, const float* S, const float* centroids, void* out,
                        float* logits, int num_splits, void* workspace, size_t ws_bytes,
                        void* stream, bool prep, bool partial, bool combine, const char* name) {
  DecodePlan P;
  int st = decode_plan(c, Q, Hq, softmax_scale, Pi, S, centroids, out, num_splits, workspace,
                       ws_bytes, prep, partial, combine, name, P);
  if (st != TQ_OK) return st;
  st = check_pending(name);
  if (st != TQ_OK) return st;
  return decode_launch(c, P, Q, Hq, softmax_scale, Pi, S, centroids, out, logits,
                       static_cast<cudaStream_t>(stream), prep, partial, combine, name);
}

int tq_decode_attention(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                        const float* Pi, const float* S, const float* centroids, void* out,
                        float* logits, int num_splits, void* workspace, size_t ws_bytes,
                        void* stream) {
  TQ_FAULT_POINT("tq_decode_attention");
  return decode_stage(c, Q, Hq, softmax_scale, Pi, S, centroids, out, logits, num_splits,
                      workspace, ws_bytes, stream, true, true, true, "tq_decode_attention");
}

int tq_decode_step(tq_cache* c, const void* K, const void* V, int64_t n_new, const void* Q, int Hq,
                   float softmax_scale, const float* Pi, const float* S, const float* T,
                   const float* centroids, const float* boundaries, void* out, float* logits,
                   int num_splits, void* workspace, size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_decode_step");
  int st = check_cache(c);
  if (st != TQ_OK) return st;
  if (n_new < 0) return fail(TQ_ERR_INVALID_ARG, "n_new=%lld", (long long)n_new);
  const tq_cache_desc& dsc = c->desc;
  const tq::Geom g = tq::geom_of(c);
  const bool fusable = n_new >= 1 && n_new <= 8 && n_new <= dsc.W && dsc.Hkv > 0 &&
                       Hq % dsc.Hkv == 0 && tq::decode_mma_supported(g, Hq / dsc.Hkv);
  if (!fusable) {
    st = tq_append(c, K, V, n_new, Pi, T, centroids, boundaries, stream);
    if (st != TQ_OK) return st;
    return tq_decode_attention(c, Q, Hq, softmax_scale, Pi, S, centroids, out, logits, num_splits,
                               workspace, ws_bytes, stream);
  }
  int64_t c_old = 0, c_new = 0;
  st = append_checks(c, K, V, n_new, Pi, T, centroids, boundaries, &c_old, &c_new);
  if (st != TQ_OK) return st;
  const int64_t n_old = c->n_total, n_tot = n_old + n_new;
  tq_cache after = *c;            // the decode reads the cache as the append leaves it
  after.n_total = n_tot;
  DecodePlan P;
  st = decode_plan(&after, Q, Hq, softmax_scale, Pi, S, centroids, out, num_splits, workspace,
                   ws_bytes, true, true, true, "tq_decode_step", P);
  if (st != TQ_OK) return st;
  st = check_pending("tq_decode_step");
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nq = c_new - c_old;
  tq::QuantSrc src{K, V, nq, c_old, n_old, n_new};
  cudaError_t e = tq::launch_decode_step_pre(src, n_new - nq, g, static_cast<uint8_t*>(c->base), Pi, T,
                                             centroids, boundaries, Q, Hq, S, softmax_scale, P.ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_step: quantise + prepare");
  c->n_total = n_tot;
  // the fused quantise writes the packed blocks from the one holding token c_old on
  return decode_launch(c, P, Q, Hq, softmax_scale, Pi, S, centroids, out, logits, s, false, true,
                       true, "tq_decode_step", c_old / tq::kBlockTokens);
}

int tq_decode_prep(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                   const float* Pi, const float* S, const float* centroids, int num_splits,
                   void* workspace, size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_decode_prep");
  return decode_stage(c, Q, Hq, softmax_scale, Pi, S, centroids, nullptr, nullptr, num_splits,
                      workspace, ws_bytes, stream, true, false, false, "tq_decode_prep");
}

int tq_decode_partial(const tq_cache* c, int Hq, float softmax_scale, const float* centroids,
                      float* logits, void* out, int num_splits, void* workspace, size_t ws_bytes,
                      void* stream) {
  TQ_FAULT_POINT("tq_decode_partial");
  return decode_stage(c, nullptr, Hq, softmax_scale, nullptr, nullptr, centroids, out, logits,
                      num_splits, workspace, ws_bytes, stream, false, true, out != nullptr,
                      "tq_decode_partial");
}

int tq_decode_combine(const tq_cache* c, int Hq, void* out, int num_splits, void* workspace,
                      size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_decode_combine");
  return decode_stage(c, nullptr, Hq, 1.f, nullptr, nullptr, nullptr, out, nullptr, num_splits,
                      workspace, ws_bytes, stream, false, false, true, "tq_decode_combine");
}

int tq_decode_partials_view(const tq_cache* c, int Hq, int num_splits, void* workspace,
                            size_t ws_bytes, float** part_ml, float** part_o, int* splits) {
  int st = check_decode_common(c, Hq, num_splits);
  if (st != TQ_OK) return st;
  if (!part_ml || !part_o || !splits)
    return fail(TQ_ERR_INVALID_ARG, "tq_decode_partials_view: null output pointer");
  const tq::Geom g = tq::geom_of(c);
  const int s = eff_splits(g, Hq / c->desc.Hkv, n_comp_of(c), num_splits);
  if (!workspace || ws_bytes < tq::decode_ws_bytes(g, Hq, s))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode_partials_view: workspace too small");
  const tq::DecodeWs ws = tq::decode_ws_carve(workspace, g, Hq, s);
  *part_ml = ws.part_ml;
  *part_o = ws.part_o;
  *splits = s;
  return ok();
}

int tq_merge_partials(const float* part_ml, const float* part_o, int64_t rows, int slots, int d,
                      int dtype, void* out, void* stream) {
  TQ_FAULT_POINT("tq_merge_partials");
  if (!part_ml || !part_o || !out) return fail(TQ_ERR_INVALID_ARG, "tq_merge_partials: null pointer");
  if (rows < 1 || rows > ((int64_t)1 << 31) - 1 || slots < 1 || d < 1 || d > 1024)
    return fail(TQ_ERR_INVALID_ARG, "tq_merge_partials: rows=%lld slots=%d d=%d", (long long)rows,
                slots, d);
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16)
    return fail(TQ_ERR_INVALID_ARG, "tq_merge_partials: dtype %d", dtype);
  int st = check_pending("tq_merge_partials");
  if (st != TQ_OK) return st;
  // the decode merge kernel over an explicit partial array: rows x 1 "heads"
  tq::Geom g{};
  g.B = (int)rows;
  g.d = d;
  g.dtype = dtype;
  tq::DecodeWs ws{};
  ws.part_ml = const_cast<float*>(part_ml);
  ws.part_o = const_cast<float*>(part_o);
  cudaError_t e = tq::launch_decode_combine(g, 1, out, slots, ws, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_merge_partials");
  return ok();
}

int tq_decode_check(const tq_cache* c, int Hq, int num_splits, const void* workspace,
                    size_t ws_bytes, void* stream) {
  int st = check_decode_common(c, Hq, num_splits);
  if (st != TQ_OK) return st;
  tq::Geom g = tq::geom_of(c);
  const int splits = eff_splits(g, Hq / c->desc.Hkv, n_comp_of(c), num_splits);
  if (!workspace) {       // the static scratch of tq_decode_attention_noalloc
    void* p = nullptr;
    st = tq::noalloc_scratch(&p);
    if (st != TQ_OK) return st;
    workspace = p;
    ws_bytes = (size_t)TQ_NOALLOC_SCRATCH_BYTES;
  }
  if (ws_bytes < tq::decode_ws_bytes(g, Hq, splits))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode_check: workspace too small");
  tq::DecodeWs ws = tq::decode_ws_carve(const_cast<void*>(workspace), g, Hq, splits);
  int flag = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&flag, ws.err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_check");
  if (flag) return fail(TQ_ERR_CUDA, "decode: a staged load did not complete within its wait limit");
  return ok();
}

// ---------------------------------------------------------------- chunked prefill
struct PrefillPlan {
  tq::Geom g, gv;          // cache geometry; virtual batch B * n
  int splits = 1, nslots = 2;
  bool mma = false;
  tq::DecodeWs ws{};
};

static int prefill_splits(const tq::Geom& g, int G, int n, bool mma, int num_splits,
                          int64_t n_comp) {
  const int64_t nblk = (n_comp + tq::kBlockTokens - 1) / tq::kBlockTokens;
  int s = num_splits > 0 ? num_splits : tq::prefill_auto_splits(g, G, n_comp, n, mma);
  if (nblk == 0) return 1;
  if (mma && tq::prefill_tc_supported(g, G, n)) {
    // the tcgen05 partial splits whole 128-token tiles and runs empty splits as
    // empty partials: any count up to the tile count (monotone in n_comp)
    const int64_t ntiles = (nblk + 1) / 2;
    return (int)(s < ntiles ? s : ntiles);
  }
  if (s > nblk) s = (int)nblk;
  const int64_t bps = (nblk + s - 1) / s;
  return (int)((nblk + bps - 1) / bps);
}

static int prefill_common(const tq_cache* c, int Hq, int n, int num_splits, const char* name) {
  int st = check_decode_common(c, Hq, num_splits);
  if (st != TQ_OK) return st;
  if (n < 1 || n > 65535) return fail(TQ_ERR_INVALID_ARG, "%s: n=%d (1..65535)", name, n);
  if ((int64_t)c->desc.B * n > (int64_t)1 << 24)
    return fail(TQ_ERR_UNSUPPORTED, "%s: B * n = %lld query tokens", name, (long long)c->desc.B * n);
  return TQ_OK;
}

static tq::Geom virtual_geom(const tq_cache* c, int n) {
  tq::Geom gv = tq::geom_of(c);
  gv.B = c->desc.B * n;
  return gv;
}

size_t tq_prefill_workspace_bytes(const tq_cache* c, int Hq, int n, int num_splits) {
  if (prefill_common(c, Hq, n, num_splits, "tq_prefill_workspace_bytes") != TQ_OK) return 0;
  const tq::Geom g = tq::geom_of(c);
  const int G = Hq / c->desc.Hkv;
  const bool mma = tq::prefill_mma_supported(g, G);
  // the split count at full capacity bounds the one any later length needs
  const int s = prefill_splits(g, G, n, mma, num_splits, c->desc.capacity);
  const int smax = num_splits > 0 ? num_splits : s;
  return tq::decode_ws_bytes(virtual_geom(c, n), Hq, smax + 1);
}

static int prefill_plan(const tq_cache* c, const void* Q, int Hq, int n, const void* K,
                        const void* V, float softmax_scale, const float* Pi, const float* S,
                        const float* centroids, void* out, int num_splits, void* workspace,
                        size_t ws_bytes, const char* name, PrefillPlan& P) {
  int st = prefill_common(c, Hq, n, num_splits, name);
  if (st != TQ_OK) return st;
  const tq_cache_desc& dsc = c->desc;
  P.g = tq::geom_of(c);
  P.gv = virtual_geom(c, n);
  const int G = Hq / dsc.Hkv;
  P.mma = tq::prefill_mma_supported(P.g, G);
  if (!P.mma && (int64_t)P.gv.B * dsc.Hkv > 65535)
    return fail(TQ_ERR_UNSUPPORTED, "%s: B * n * Hkv = %lld above 65535 on this shape's path", name,
                (long long)P.gv.B * dsc.Hkv);
  P.splits = prefill_splits(P.g, G, n, P.mma, num_splits, n_comp_of(c));
  P.nslots = P.splits + 1;
  const size_t need = tq::decode_ws_bytes(P.gv, Hq, P.nslots);
  if (!workspace || !aligned16(workspace) || ws_bytes < need)
    return fail(TQ_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed", name, need);
  if (!Q || !K || !V || !out || !S || !aligned16(S) || (dsc.b1 > 0 && (!Pi || !aligned16(Pi))))
    return fail(TQ_ERR_INVALID_ARG, "%s: Q, K, V, out, S (and Pi when b1>0) needed", name);
  if (!std::isfinite(softmax_scale)) return fail(TQ_ERR_INVALID_ARG, "%s: softmax_scale", name);
  if (dsc.b1 > 0 && !centroids) return fail(TQ_ERR_INVALID_ARG, "%s: centroids needed", name);
  P.ws = tq::decode_ws_carve(workspace, P.gv, Hq, P.nslots);
  return TQ_OK;
}

int tq_prefill_attention(const tq_cache* c, const void* Q, int Hq, int n, const void* K,
                         const void* V, float softmax_scale, const float* Pi, const float* S,
                         const float* centroids, void* out, int num_splits, void* workspace,
                         size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_prefill_attention");
  PrefillPlan P;
  int st = prefill_plan(c, Q, Hq, n, K, V, softmax_scale, Pi, S, centroids, out, num_splits,
                        workspace, ws_bytes, "tq_prefill_attention", P);
  if (st != TQ_OK) return st;
  st = check_pending("tq_prefill_attention");
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* base = static_cast<const uint8_t*>(c->base);
  cudaError_t e = P.mma ? tq::launch_decode_prep_mma(P.gv, Q, Hq, Pi, S, centroids, softmax_scale,
                                                     P.ws, s)
                        : tq::launch_decode_prep(P.gv, Q, Hq, Pi, S, P.ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_attention: prepare");
  const bool tc = P.mma && tq::prefill_tc_supported(P.g, Hq / c->desc.Hkv, n);
  e = tc      ? tq::launch_prefill_partial_tc(P.g, base, c->n_total, Hq, n, P.splits, P.nslots,
                                              centroids, P.ws, s)
    : P.mma ? tq::launch_prefill_partial_mma(P.g, base, c->n_total, Hq, n, P.splits, P.nslots, P.ws, s)
            : tq::launch_decode_partial(P.gv, base, c->n_total, Hq, softmax_scale, centroids, nullptr,
                                        P.splits, P.ws, s, n, P.nslots, false);
  if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_attention: history");
  e = tq::launch_prefill_exact(P.g, base, c->n_total, Hq, n, K, V, softmax_scale, P.nslots,
                               P.splits, P.ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_attention: exact segment");
  e = tq::launch_decode_combine(P.gv, Hq, out, P.nslots, P.ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_attention: combine");
  return ok();
}

int tq_prefill_check(const tq_cache* c, int Hq, int n, int num_splits, const void* workspace,
                     size_t ws_bytes, void* stream) {
  int st = prefill_common(c, Hq, n, num_splits, "tq_prefill_check");
  if (st != TQ_OK) return st;
  const tq::Geom g = tq::geom_of(c);
  const tq::Geom gv = virtual_geom(c, n);
  const int G = Hq / c->desc.Hkv;
  const int splits = prefill_splits(g, G, n, tq::prefill_mma_supported(g, G), num_splits,
                                    n_comp_of(c));
  if (!workspace || ws_bytes < tq::decode_ws_bytes(gv, Hq, splits + 1))
    return fail(TQ_ERR_INVALID_ARG, "tq_prefill_check: workspace too small");
  tq::DecodeWs ws = tq::decode_ws_carve(const_cast<void*>(workspace), gv, Hq, splits + 1);
  int flag = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&flag, ws.err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "tq_prefill_check");
  if (flag) return fail(TQ_ERR_CUDA, "prefill: a staged load did not complete within its wait limit");
  return ok();
}

int tq_quantize_check(void* stream) {
  int flag = 0;
  cudaError_t e = tq::quantize_error_flag(&flag, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_quantize_check");
  if (flag) return fail(TQ_ERR_CUDA, "quantise: a tensor-core product did not complete within its wait limit");
  return ok();
}

static int parse_list(const char* s, int* out, int max_n) {
  int n = 0;
  const char* p = s;
  while (*p) {
    while (*p && std::isspace((unsigned char)*p)) ++p;
    if (!*p) break;
    char* end = nullptr;
    long v = std::strtol(p, &end, 10);
    if (end == p || v < 0 || v > 1000000) return -1;
    if (n >= max_n) return -1;
    out[n++] = (int)v;
    p = end;
    while (*p && std::isspace((unsigned char)*p)) ++p;
    if (*p == ',') {
      ++p;
      continue;
    }
    if (*p) return -1;
  }
  return n;
}

size_t tq_key_moments_workspace_bytes(void) { return tq::key_moments_ws_bytes(); }

int tq_key_moments(const void* K, int dtype, int64_t n, double* out, void* workspace,
                   size_t ws_bytes, void* stream) {
  TQ_FAULT_POINT("tq_key_moments");
  if (!K || !out || !aligned16(K)) return fail(TQ_ERR_INVALID_ARG, "tq_key_moments: K (16-byte aligned) and out needed");
  if (n < 1) return fail(TQ_ERR_INVALID_ARG, "tq_key_moments: n=%lld", (long long)n);
  if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16)
    return fail(TQ_ERR_INVALID_ARG, "tq_key_moments: dtype %d", dtype);
  if (!workspace || !aligned16(workspace) || ws_bytes < tq::key_moments_ws_bytes())
    return fail(TQ_ERR_INVALID_ARG, "tq_key_moments: workspace of %zu bytes needed",
                tq::key_moments_ws_bytes());
  int st = check_pending("tq_key_moments");
  if (st != TQ_OK) return st;
  cudaError_t e = tq::launch_key_moments(K, dtype, n, out, static_cast<double*>(workspace),
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_key_moments");
  return ok();
}

int tq_sensitivity_profile(const double* layer_var, int L, int num_groups, int m_avg, int m_min,
                           int m_max, tq_layer_groups* out) {
  if (!layer_var || !out) return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: null argument");
  if (L < 1 || num_groups < 1 || num_groups > 8 || num_groups > L)
    return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: L=%d num_groups=%d (1..min(8, L))", L,
                num_groups);
  if (!valid_m(m_min) || !valid_m(m_max) || m_min > m_max)
    return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: m range [%d, %d]", m_min, m_max);
  if (m_avg < m_min) return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: m_avg=%d below m_min", m_avg);
  for (int i = 0; i < L; ++i)
    if (!std::isfinite(layer_var[i]) || layer_var[i] < 0.0)
      return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: variance of layer %d", i);
  tq_layer_groups g;
  std::memset(&g, 0, sizeof(g));
  tq::sensitivity_segment(layer_var, L, num_groups, g.bound);
  if (tq::sensitivity_allocate(layer_var, L, g.bound, num_groups, m_avg, m_min, m_max, g.m) != 0)
    return fail(TQ_ERR_INVALID_ARG, "tq_sensitivity_profile: budget below m_min");
  g.n = num_groups;
  *out = g;
  return ok();
}

int tq_layer_groups_parse(const char* boundaries, const char* sketch_dims, tq_layer_groups* out) {
  if (!boundaries || !sketch_dims || !out) return fail(TQ_ERR_INVALID_ARG, "null argument");
  tq_layer_groups g;
  std::memset(&g, 0, sizeof(g));
  int nb = parse_list(boundaries, g.bound, 7);
  int nm = parse_list(sketch_dims, g.m, 8);
  if (nb < 0 || nm < 1) return fail(TQ_ERR_INVALID_ARG, "could not parse layer groups");
  if (nm != nb + 1) return fail(TQ_ERR_INVALID_ARG, "%d sketch dims for %d boundaries", nm, nb);
  for (int i = 0; i < nb; ++i)
    if (g.bound[i] < 1 || (i > 0 && g.bound[i] <= g.bound[i - 1]))
      return fail(TQ_ERR_INVALID_ARG, "boundaries must increase from >= 1");
  for (int i = 0; i < nm; ++i)
    if (!valid_m(g.m[i])) return fail(TQ_ERR_INVALID_ARG, "sketch dim %d invalid", g.m[i]);
  g.n = nm;
  *out = g;
  return ok();
}

int tq_m_for_layer(const tq_layer_groups* g, int layer) {
  if (!g || g->n < 1 || g->n > 8 || layer < 0) return -1;
  int k = 0;
  while (k < g->n - 1 && layer >= g->bound[k]) ++k;
  return g->m[k];
}

}  // extern "C"
