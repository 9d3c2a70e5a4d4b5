// C ABI of libtq: argument checking, context construction and kernel dispatch.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.cuh"

namespace tq {

namespace {
thread_local std::string g_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_ns{2000000000ull};
std::atomic<int> g_stall{0};
std::atomic<int> g_fail_alloc{-1};     // index of the tq_init allocation to fail (-1: none)
std::atomic<int> g_alloc_count{0};
}  // namespace

uint64_t pipeline_wait_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
bool debug_stall() { return g_stall.load(std::memory_order_relaxed) != 0; }

cudaError_t dev_alloc(void** p, size_t bytes) {
  const int i = g_alloc_count.fetch_add(1, std::memory_order_relaxed);
  if (i == g_fail_alloc.load(std::memory_order_relaxed)) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}

// NVTX range around each entry point (a no-op unless a profiler is attached).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

void set_error(const std::string& msg) { g_error = msg; }

int fail(int code, const std::string& msg) {
  g_error = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  g_error = std::string(what) + ": " + cudaGetErrorString(e);
  return TQ_ERR_CUDA;
}

void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return TQ_OK;
}

namespace {

int check_device(const tq_ctx* ctx) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != ctx->device) return fail(TQ_ERR_INVALID_ARG, "context belongs to another CUDA device than the current one");
  return TQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_packed(const tq_ctx* ctx, const tq_packed* pk, const char* name) {
  if (!pk) return fail(TQ_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!pk->codes || !pk->norm) return fail(TQ_ERR_INVALID_ARG, std::string(name) + ": codes/norm pointer is NULL");
  if (ctx->mode == TQ_MODE_PROD && !pk->rnorm)
    return fail(TQ_ERR_INVALID_ARG, std::string(name) + ": rnorm is required for a prod-mode context");
  if (pk->cap < 0) return fail(TQ_ERR_INVALID_ARG, std::string(name) + ": negative capacity");
  if (!aligned(pk->codes, 16)) return fail(TQ_ERR_UNSUPPORTED, std::string(name) + ": codes must be 16-byte aligned");
  return TQ_OK;
}

int alloc_copy(float** dst, const std::vector<double>& src) {
  std::vector<float> f(src.size());
  for (size_t i = 0; i < src.size(); ++i) f[i] = (float)src[i];
  cudaError_t e = dev_alloc(reinterpret_cast<void**>(dst), f.size() * sizeof(float));
  if (e != cudaSuccess) {
    *dst = nullptr;
    return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  }
  e = cudaMemcpy(*dst, f.data(), f.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(params)");
  return TQ_OK;
}

std::vector<double> transpose(const std::vector<double>& a, int rows, int cols) {
  std::vector<double> t((size_t)rows * cols);
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < cols; ++j) t[(size_t)j * rows + i] = a[(size_t)i * cols + j];
  return t;
}

// bf16 / fp16 splits of the tensor-core operands: Pi = hi + mid + lo (bf16, ~24 bits),
// 16*M = hi + lo (fp16, ~22 bits); each split row-major [d][d].
int alloc_splits(tq_ctx* c) {
  const HostParams& h = c->host;
  const int d = c->lay.d;
  const size_t nn = (size_t)d * d;
  std::vector<__nv_bfloat16> pis(3 * nn);
  for (size_t i = 0; i < nn; ++i) {
    double v = h.Pi[i];
    __nv_bfloat16 a = __float2bfloat16_rn((float)v);
    double r1 = v - (double)__bfloat162float(a);
    __nv_bfloat16 b = __float2bfloat16_rn((float)r1);
    double r2 = r1 - (double)__bfloat162float(b);
    pis[i] = a;
    pis[nn + i] = b;
    pis[2 * nn + i] = __float2bfloat16_rn((float)r2);
  }
  cudaError_t e = dev_alloc(&c->Pi_split, pis.size() * sizeof(__nv_bfloat16));
  if (e != cudaSuccess) return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  e = cudaMemcpy(c->Pi_split, pis.data(), pis.size() * sizeof(__nv_bfloat16), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(Pi splits)");
  if (c->mode == TQ_MODE_PROD) {
    std::vector<__half> ms(2 * nn);
    for (size_t i = 0; i < nn; ++i) {
      double v = 16.0 * h.M[i];
      __half a = __float2half_rn((float)v);
      ms[i] = a;
      ms[nn + i] = __float2half_rn((float)(v - (double)__half2float(a)));
    }
    e = dev_alloc(&c->M_split, ms.size() * sizeof(__half));
    if (e != cudaSuccess) return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
    e = cudaMemcpy(c->M_split, ms.data(), ms.size() * sizeof(__half), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(M splits)");
  }
  return TQ_OK;
}

// Dequantize operands (d <= 128): B[n][k] = 16 A[k][n] * scale as fp16 hi + lo, [2][N][d_pad],
// for A = Pi (plain reconstruction) and A = S with scale sqrt(pi/2)/m (QJL term).
int alloc_dequant_operand(void** dst, const std::vector<double>& A, int d, int d_pad, double scale) {
  const int K = d_pad, N = 16 * ((d + 15) / 16);
  std::vector<__half> b((size_t)2 * N * K, __float2half(0.f));
  for (int n = 0; n < d; ++n)
    for (int k = 0; k < d; ++k) {
      const double v = 16.0 * scale * A[(size_t)k * d + n];
      const __half h = __float2half_rn((float)v);
      b[(size_t)n * K + k] = h;
      b[(size_t)N * K + (size_t)n * K + k] = __float2half_rn((float)(v - (double)__half2float(h)));
    }
  cudaError_t e = dev_alloc(dst, b.size() * sizeof(__half));
  if (e != cudaSuccess) return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  e = cudaMemcpy(*dst, b.data(), b.size() * sizeof(__half), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(dequantize operand)");
  return TQ_OK;
}

// Projection operands of the workspace quantize path: 16 Pi and 16 M as fp16 hi + lo,
// [2][d_pad][K] (K = 64 ceil(d/64)), zero padded.
int alloc_projection(void** dst, const std::vector<double>& A, int d, int d_pad) {
  const int K = 64 * ((d + 63) / 64);
  std::vector<__half> b((size_t)2 * d_pad * K, __float2half(0.f));
  for (int n = 0; n < d; ++n)
    for (int k = 0; k < d; ++k) {
      const double v = 16.0 * A[(size_t)n * d + k];
      const __half h = __float2half_rn((float)v);
      b[(size_t)n * K + k] = h;
      b[(size_t)d_pad * K + (size_t)n * K + k] = __float2half_rn((float)(v - (double)__half2float(h)));
    }
  cudaError_t e = dev_alloc(dst, b.size() * sizeof(__half));
  if (e != cudaSuccess) return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  e = cudaMemcpy(*dst, b.data(), b.size() * sizeof(__half), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(projection operand)");
  return TQ_OK;
}

void release(tq_ctx* c) {
  if (!c) return;
  cudaFree(c->Pi16);
  cudaFree(c->M16);
  cudaFree(c->PiT_f16);
  cudaFree(c->ST_f16);
  cudaFree(c->Pi_split);
  cudaFree(c->M_split);
  cudaFree(c->dev_err);
  cudaFree(c->Pi);
  cudaFree(c->PiT);
  cudaFree(c->ST);
  delete c;
}

int check_args_common(int d, int bits, int mode) {
  if (mode != TQ_MODE_PROD && mode != TQ_MODE_MSE) return fail(TQ_ERR_INVALID_ARG, "mode must be TQ_MODE_PROD or TQ_MODE_MSE");
  if (d < 3 || d > 4096) return fail(TQ_ERR_UNSUPPORTED, "d must be in [3, 4096]");
  if (mode == TQ_MODE_PROD && (bits < 2 || bits > 5)) return fail(TQ_ERR_UNSUPPORTED, "prod mode needs bits in [2, 5]");
  if (mode == TQ_MODE_MSE && (bits < 1 || bits > 4)) return fail(TQ_ERR_UNSUPPORTED, "MSE mode needs bits in [1, 4]");
  return TQ_OK;
}

}  // namespace

// Every argument check of tq_decode_attention except the workspace size (shared with
// tq_decode_attention_static, which checks its own scratch size after these).
int check_decode_args(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off, int ngroups,
                      const void* q, int q_dtype, const tq_packed* kcache, const tq_packed* vcache,
                      const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len, const float* out,
                      int page) {
  if (!kctx || !vctx || !group_off || !kcache || !vcache) return fail(TQ_ERR_INVALID_ARG, "NULL argument");
  if (ngroups < 1 || ngroups > 4) return fail(TQ_ERR_UNSUPPORTED, "ngroups must be in [1, 4]");
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_len < 0) return fail(TQ_ERR_INVALID_ARG, "bad sizes");
  if (Hq % Hkv != 0) return fail(TQ_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (q_dtype != TQ_DTYPE_F32 && q_dtype != TQ_DTYPE_BF16) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be F32 or BF16");
  if (group_off[0] != 0 || group_off[ngroups] != D) return fail(TQ_ERR_INVALID_ARG, "group_off must span [0, D]");
  if (B == 0) return TQ_OK;
  if (!q || !seq_lens || !out) return fail(TQ_ERR_INVALID_ARG, "NULL q, seq_lens or out");
  for (int g = 0; g < ngroups; ++g) {
    const tq_ctx* kc = kctx[g];
    const tq_ctx* vc = vctx[g];
    if (!kc || !vc) return fail(TQ_ERR_INVALID_ARG, "NULL context");
    int w = group_off[g + 1] - group_off[g];
    if (w <= 0) return fail(TQ_ERR_INVALID_ARG, "group_off must be increasing");
    if (kc->mode != TQ_MODE_PROD || vc->mode != TQ_MODE_MSE)
      return fail(TQ_ERR_INVALID_ARG, "key contexts must be prod mode, value contexts MSE mode");
    if (kc->lay.d != w || vc->lay.d != w) return fail(TQ_ERR_INVALID_ARG, "context dimension differs from its group width");
    int r = check_packed(kc, &kcache[g], "kcache");
    if (r != TQ_OK) return r;
    if ((r = check_packed(vc, &vcache[g], "vcache")) != TQ_OK) return r;
    // contiguous caches hold every (sequence, kv head, token) slot; paged ones at least one page
    int64_t need = page > 0 ? (int64_t)Hkv * page : (int64_t)B * Hkv * max_len;
    if (kcache[g].cap < need || vcache[g].cap < need)
      return fail(TQ_ERR_INVALID_ARG, page > 0 ? "cache capacity below one page (Hkv*page_tokens)"
                                               : "cache capacity below B*Hkv*max_len");
    if ((r = check_device(kc)) != TQ_OK) return r;
  }
  return TQ_OK;
}

}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_last_error(void) { return g_error.c_str(); }

int tq_channel_perm_by_score(const float* score, int D, int w0, int32_t* perm) {
  if (!score || !perm || D <= 0 || w0 < 0 || w0 > D) return fail(TQ_ERR_INVALID_ARG, "bad channel permutation arguments");
  std::vector<int> order(D);
  for (int i = 0; i < D; ++i) order[i] = i;
  // the w0 highest scores (ties to the lower channel) form the first group
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return score[a] > score[b]; });
  std::vector<char> first(D, 0);
  for (int i = 0; i < w0; ++i) first[order[i]] = 1;
  int p = 0;
  for (int i = 0; i < D; ++i)
    if (first[i]) perm[p++] = i;
  for (int i = 0; i < D; ++i)
    if (!first[i]) perm[p++] = i;
  return TQ_OK;
}

int tq_debug_set_wait_limit(uint64_t ns) {
  g_wait_ns.store(ns, std::memory_order_relaxed);
  return TQ_OK;
}

int tq_debug_inject_stall(int on) {
  g_stall.store(on ? 1 : 0, std::memory_order_relaxed);
  return TQ_OK;
}

int tq_debug_fail_alloc(int index) {
  g_alloc_count.store(0, std::memory_order_relaxed);
  g_fail_alloc.store(index, std::memory_order_relaxed);
  return TQ_OK;
}

uint64_t tq_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int tq_host_params(int d, int bits, uint64_t seed, int mode, double* Pi, double* S, double* centroids,
                   double* boundaries) {
  int r = check_args_common(d, bits, mode);
  if (r != TQ_OK) return r;
  HostParams p;
  if (!build_params(d, bits, seed, mode, &p)) return fail(TQ_ERR_INVALID_ARG, "bad parameters");
  if (Pi) std::memcpy(Pi, p.Pi.data(), p.Pi.size() * sizeof(double));
  if (S && mode == TQ_MODE_PROD) std::memcpy(S, p.S.data(), p.S.size() * sizeof(double));
  if (centroids) std::memcpy(centroids, p.centroids.data(), p.centroids.size() * sizeof(double));
  if (boundaries) std::memcpy(boundaries, p.boundaries.data(), p.boundaries.size() * sizeof(double));
  return TQ_OK;
}

int tq_init(tq_ctx** out, int d, int bits, uint64_t seed, int mode) {
  Range range_("tq_init");
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  int r = check_args_common(d, bits, mode);
  if (r != TQ_OK) return r;
  tq_ctx* c = new (std::nothrow) tq_ctx();
  if (!c) return fail(TQ_ERR_ALLOC, "host allocation failed");
  cudaError_t e = cudaGetDevice(&c->device);
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "cudaGetDevice");
  }
  if (!build_params(d, bits, seed, mode, &c->host)) {
    delete c;
    return fail(TQ_ERR_INVALID_ARG, "bad parameters");
  }
  const HostParams& h = c->host;
  c->mode = mode;
  c->bits = bits;
  c->m = h.m;
  Layout& L = c->lay;
  L.d = d;
  L.k = h.k;
  L.d_pad = ((d + 31) / 32) * 32;
  L.planes = h.k + (mode == TQ_MODE_PROD ? 1 : 0);
  L.code_bytes = L.planes * L.d_pad / 8;
  Codebook& cb = c->cb;
  cb.K = 1 << h.k;
  for (int j = 0; j < kMaxLevels; ++j) {
    cb.c[j] = j < cb.K ? (float)h.centroids[j] : 0.f;
    cb.t[j] = j < cb.K - 1 ? (float)h.boundaries[j] : INFINITY;
  }
  for (int code = 0; code < kMaxLevels; ++code) cb.cc[code] = code < cb.K ? cb.c[code_index(code, h.k)] : 0.f;
  c->sqrt_pi_over_2_over_m = mode == TQ_MODE_PROD ? (float)(std::sqrt(M_PI / 2.0) / h.m) : 0.f;
  for (int j = 0; j < h.m; ++j) {
    double r = 0.0;
    for (int i = 0; i < d; ++i) r += h.S[(size_t)j * d + i] * h.S[(size_t)j * d + i];
    c->s_rowmax = std::max(c->s_rowmax, (float)(std::sqrt(r) * (1.0 + 1e-6)));
  }
  if ((r = alloc_copy(&c->Pi, h.Pi)) != TQ_OK || (r = alloc_copy(&c->PiT, transpose(h.Pi, d, d))) != TQ_OK) {
    release(c);
    return r;
  }
  if (mode == TQ_MODE_PROD) {
    if ((r = alloc_copy(&c->ST, transpose(h.S, h.m, d))) != TQ_OK) {
      release(c);
      return r;
    }
  }
  if (d == 64 || d == 128) {
    if ((r = alloc_splits(c)) != TQ_OK) {
      release(c);
      return r;
    }
  }
  if (d <= 128 && ((r = alloc_dequant_operand(&c->PiT_f16, h.Pi, d, L.d_pad, 1.0)) != TQ_OK ||
                    (mode == TQ_MODE_PROD &&
                     (r = alloc_dequant_operand(&c->ST_f16, h.S, d, L.d_pad, std::sqrt(M_PI / 2.0) / h.m)) != TQ_OK))) {
    release(c);
    return r;
  }
  if ((r = alloc_projection(&c->Pi16, h.Pi, d, L.d_pad)) != TQ_OK ||
      (mode == TQ_MODE_PROD && (r = alloc_projection(&c->M16, h.M, d, L.d_pad)) != TQ_OK)) {
    release(c);
    return r;
  }
  e = dev_alloc(reinterpret_cast<void**>(&c->dev_err), sizeof(int));
  if (e != cudaSuccess) {
    release(c);
    return fail(TQ_ERR_ALLOC, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  }
  e = cudaMemset(c->dev_err, 0, sizeof(int));
  if (e != cudaSuccess) {
    release(c);
    return cuda_fail(e, "cudaMemset(error word)");
  }
  *out = c;
  return TQ_OK;
}

int tq_get_device_error(const tq_ctx* ctx, int* code) {
  if (!ctx || !code) return fail(TQ_ERR_INVALID_ARG, "NULL argument");
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, ctx->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
  *code = v;
  if (v != 0) {
    e = cudaMemset(ctx->dev_err, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error word)");
  }
  return TQ_OK;
}

void tq_free(tq_ctx* ctx) { release(ctx); }

int tq_get_info(const tq_ctx* ctx, tq_info* info) {
  if (!ctx || !info) return fail(TQ_ERR_INVALID_ARG, "NULL argument");
  info->d = ctx->lay.d;
  info->bits = ctx->bits;
  info->k = ctx->lay.k;
  info->m = ctx->m;
  info->mode = ctx->mode;
  info->planes = ctx->lay.planes;
  info->d_pad = ctx->lay.d_pad;
  info->code_bytes = ctx->lay.code_bytes;
  info->seed = ctx->host.seed;
  return TQ_OK;
}

int tq_get_params(const tq_ctx* ctx, double* Pi, double* S, double* centroids, double* boundaries) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  const HostParams& h = ctx->host;
  if (Pi) std::memcpy(Pi, h.Pi.data(), h.Pi.size() * sizeof(double));
  if (S && ctx->mode == TQ_MODE_PROD) std::memcpy(S, h.S.data(), h.S.size() * sizeof(double));
  if (centroids) std::memcpy(centroids, h.centroids.data(), h.centroids.size() * sizeof(double));
  if (boundaries) std::memcpy(boundaries, h.boundaries.data(), h.boundaries.size() * sizeof(double));
  return TQ_OK;
}

size_t tq_quantize_workspace_size(const tq_ctx* ctx, int x_dtype, int64_t n, int64_t ld) {
  if (!ctx || n < 0) return 0;
  if (n == 0 || quantize_tc_applies(ctx, x_dtype, n, ld)) return 0;
  return quantize_gen_workspace(ctx, n);
}

static int quantize_common(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const int32_t* cols,
                           const tq_packed* dst, const int64_t* dst_slot, void* workspace, size_t ws_bytes,
                           tq_stream_t stream) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && !x) return fail(TQ_ERR_INVALID_ARG, "x is NULL");
  if (ld < ctx->lay.d) return fail(TQ_ERR_INVALID_ARG, "ld < d");
  if (x_dtype != TQ_DTYPE_F32 && x_dtype != TQ_DTYPE_BF16 && x_dtype != TQ_DTYPE_F16)
    return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_DTYPE_F32, BF16 or F16");
  int r = check_packed(ctx, dst, "dst");
  if (r != TQ_OK) return r;
  if (!dst_slot && n > dst->cap) return fail(TQ_ERR_INVALID_ARG, "n exceeds dst->cap");
  if ((r = check_device(ctx)) != TQ_OK) return r;
  if (n == 0) return TQ_OK;
  if (cols)
    return launch_quantize_gen(ctx, x, x_dtype, n, ld, cols, dst, dst_slot, workspace, ws_bytes, (cudaStream_t)stream);
  return launch_quantize(ctx, x, x_dtype, n, ld, dst, dst_slot, workspace, ws_bytes, (cudaStream_t)stream);
}

int tq_quantize_kv(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                   const int64_t* dst_slot, void* workspace, size_t ws_bytes, tq_stream_t stream) {
  Range range_("tq_quantize_kv");
  return quantize_common(ctx, x, x_dtype, n, ld, nullptr, dst, dst_slot, workspace, ws_bytes, stream);
}

size_t tq_quantize_cols_workspace_size(const tq_ctx* ctx, int64_t n) {
  if (!ctx || n <= 0) return 0;
  return quantize_gen_workspace(ctx, n);
}

int tq_quantize_kv_cols(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const int32_t* cols,
                        const tq_packed* dst, const int64_t* dst_slot, void* workspace, size_t ws_bytes,
                        tq_stream_t stream) {
  Range range_("tq_quantize_kv_cols");
  if (!cols) return fail(TQ_ERR_INVALID_ARG, "cols is NULL");
  return quantize_common(ctx, x, x_dtype, n, ld, cols, dst, dst_slot, workspace, ws_bytes, stream);
}

static int dequantize_common(const tq_ctx* ctx, const tq_packed* src, const int64_t* src_slot, int64_t n, float* out,
                             int64_t ld, bool qjl, tq_stream_t stream) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && !out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if (ld < ctx->lay.d) return fail(TQ_ERR_INVALID_ARG, "ld < d");
  if (qjl && ctx->mode != TQ_MODE_PROD) return fail(TQ_ERR_INVALID_ARG, "the QJL reconstruction needs a prod-mode context");
  int r = check_packed(ctx, src, "src");
  if (r != TQ_OK) return r;
  if (!src_slot && n > src->cap) return fail(TQ_ERR_INVALID_ARG, "n exceeds src->cap");
  if ((r = check_device(ctx)) != TQ_OK) return r;
  return launch_dequantize_tc(ctx, src, src_slot, n, out, ld, qjl, (cudaStream_t)stream);
}

int tq_dequantize(const tq_ctx* ctx, const tq_packed* src, const int64_t* src_slot, int64_t n, float* out,
                  int64_t ld, tq_stream_t stream) {
  Range range_("tq_dequantize");
  return dequantize_common(ctx, src, src_slot, n, out, ld, false, stream);
}

int tq_dequantize_qjl(const tq_ctx* ctx, const tq_packed* src, const int64_t* src_slot, int64_t n, float* out,
                      int64_t ld, tq_stream_t stream) {
  Range range_("tq_dequantize_qjl");
  return dequantize_common(ctx, src, src_slot, n, out, ld, true, stream);
}

int tq_prepare_queries(const tq_ctx* ctx, const float* q, int64_t nq, int64_t ld, float* out, tq_stream_t stream) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (nq < 0) return fail(TQ_ERR_INVALID_ARG, "nq < 0");
  if (nq > 0 && (!q || !out)) return fail(TQ_ERR_INVALID_ARG, "NULL q or out");
  if (ld < ctx->lay.d) return fail(TQ_ERR_INVALID_ARG, "ld < d");
  int r = check_device(ctx);
  if (r != TQ_OK) return r;
  return launch_prepare_queries(ctx, q, TQ_DTYPE_F32, nq, ld, out, ctx->lay.d + ctx->m, (cudaStream_t)stream);
}

size_t tq_attn_logits_workspace_size(const tq_ctx* ctx, int64_t nq) {
  if (!ctx || nq < 0) return 0;
  return logits_mma_workspace(nq, ctx->lay.d);
}

int tq_attn_logits(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* logits,
                   void* workspace, size_t ws_bytes, tq_stream_t stream) {
  Range range_("tq_attn_logits");
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (nq < 0 || n < 0) return fail(TQ_ERR_INVALID_ARG, "negative size");
  if (nq > 0 && (!q || !logits) && n > 0) return fail(TQ_ERR_INVALID_ARG, "NULL q or logits");
  int r = check_packed(ctx, keys, "keys");
  if (r != TQ_OK) return r;
  if (n > keys->cap) return fail(TQ_ERR_INVALID_ARG, "n exceeds keys->cap");
  size_t need = tq_attn_logits_workspace_size(ctx, nq);
  if (need > 0 && (!workspace || ws_bytes < need)) return fail(TQ_ERR_WORKSPACE, "workspace too small");
  if ((r = check_device(ctx)) != TQ_OK) return r;
  if (nq == 0 || n == 0) return TQ_OK;
  return launch_logits(ctx, q, nq, keys, n, logits, workspace, (cudaStream_t)stream);
}

size_t tq_decode_workspace_size(int B, int Hq, int Hkv, int D, int ngroups, int64_t max_len) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || ngroups <= 0 || max_len < 0) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, D, ngroups, max_len, D);
}

int tq_decode_attention_ex(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off, int ngroups,
                           const void* q, int q_dtype, const tq_packed* kcache, const tq_packed* vcache,
                           const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len, float scale,
                           float* out, const tq_decode_opts* opts, void* workspace, size_t ws_bytes,
                           tq_stream_t stream) {
  Range range_("tq_decode_attention");
  const int32_t* perm = opts ? opts->channel_perm : nullptr;
  const int32_t* table = opts ? opts->block_table : nullptr;
  const int page = table ? opts->page_tokens : 0;
  if (table && (page <= 0 || page % 64 != 0 || max_len % page != 0))
    return fail(TQ_ERR_INVALID_ARG, "page_tokens must be a positive multiple of 64 that divides max_len");
  int r = check_decode_args(kctx, vctx, group_off, ngroups, q, q_dtype, kcache, vcache, seq_lens, B, Hq, Hkv, D,
                            max_len, out, page);
  if (r != TQ_OK) return r;
  if (B == 0) return TQ_OK;
  size_t need = tq_decode_workspace_size(B, Hq, Hkv, D, ngroups, max_len);
  if (!workspace || ws_bytes < need) return fail(TQ_ERR_WORKSPACE, "workspace too small");
  return launch_decode(kctx, vctx, group_off, ngroups, perm, table, page, q, q_dtype, kcache, vcache, seq_lens, B, Hq,
                       Hkv, D, max_len, scale, out, workspace, (cudaStream_t)stream);
}

int tq_decode_attention(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off, int ngroups,
                        const void* q, int q_dtype, const tq_packed* kcache, const tq_packed* vcache,
                        const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len, float scale,
                        float* out, void* workspace, size_t ws_bytes, tq_stream_t stream) {
  return tq_decode_attention_ex(kctx, vctx, group_off, ngroups, q, q_dtype, kcache, vcache, seq_lens, B, Hq, Hkv, D,
                                max_len, scale, out, nullptr, workspace, ws_bytes, stream);
}

size_t tq_search_workspace_size(const tq_ctx* ctx, int64_t nq, int64_t N, int k) {
  if (!ctx || nq < 0 || N < 0 || k < 1) return 0;
  return search_tc_workspace(ctx, nq, N, k);
}

int tq_search_topk(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                   float* scores, int64_t* ids, void* workspace, size_t ws_bytes, tq_stream_t stream) {
  Range range_("tq_search_topk");
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (ctx->mode != TQ_MODE_PROD) return fail(TQ_ERR_INVALID_ARG, "search needs a prod-mode context");
  if (nq < 0 || N < 1) return fail(TQ_ERR_INVALID_ARG, "bad sizes");
  if (k < 1 || k > 64 || k > N) return fail(TQ_ERR_UNSUPPORTED, "k must be in [1, min(64, N)]");
  int r = check_packed(ctx, db, "db");
  if (r != TQ_OK) return r;
  if (N > db->cap) return fail(TQ_ERR_INVALID_ARG, "N exceeds db->cap");
  if (nq > 0 && (!q || !scores || !ids)) return fail(TQ_ERR_INVALID_ARG, "NULL q, scores or ids");
  size_t need = tq_search_workspace_size(ctx, nq, N, k);
  if (!workspace || ws_bytes < need) return fail(TQ_ERR_WORKSPACE, "workspace too small");
  if ((r = check_device(ctx)) != TQ_OK) return r;
  return launch_search(ctx, q, nq, db, N, k, scores, ids, workspace, (cudaStream_t)stream);
}

}  // extern "C"
