// Kernel-family selection for each hot-path call.
#include "common.cuh"
#include "kernels.cuh"

#include <cstdlib>

namespace tq {

// TQ_FORCE_SIMT=1 routes every call to the CUDA-core kernels (used to cross-check the
// tensor-core kernels against the CUDA-core rung on the same inputs).
bool force_simt() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("TQ_FORCE_SIMT");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

int launch_quantize(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                    const int64_t* slots, cudaStream_t st) {
  if (!force_simt()) {
    int r = launch_quantize_tc(ctx, x, x_dtype, n, ld, dst, slots, st);
    if (r != kNotHandled) return r;
  }
  return launch_quantize_simt(ctx, x, x_dtype, n, ld, dst, slots, st);
}

int launch_logits(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* logits,
                  void* ws, cudaStream_t st) {
  if (!force_simt()) {
    int r = launch_logits_mma(ctx, q, nq, keys, n, logits, ws, st);
    if (r != kNotHandled) return r;
  }
  float* qprep = static_cast<float*>(ws);
  int r = launch_prepare_queries(ctx, q, TQ_DTYPE_F32, nq, ctx->lay.d, qprep, ctx->lay.d + ctx->m, st);
  if (r != TQ_OK) return r;
  return launch_logits_simt(ctx, qprep, nq, keys, n, logits, st);
}

int launch_decode(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G, const void* q,
                  int q_dtype, const tq_packed* kc, const tq_packed* vc, const int32_t* seq_lens, int B, int Hq,
                  int Hkv, int D, int64_t max_len, float scale, float* out, void* ws, cudaStream_t st) {
  if (!force_simt()) {
    int r = launch_decode_mma(kctx, vctx, off, G, q, q_dtype, kc, vc, seq_lens, B, Hq, Hkv, D, max_len, scale, out,
                              ws, st);
    if (r != kNotHandled) return r;
  }
  return launch_decode_simt(kctx, vctx, off, G, q, q_dtype, kc, vc, seq_lens, B, Hq, Hkv, D, max_len, scale, out, ws,
                            st);
}

int launch_search(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                  float* scores, int64_t* ids, void* ws, cudaStream_t st) {
  if (!force_simt()) {
    int r = launch_search_mma(ctx, q, nq, db, N, k, scores, ids, ws, st);
    if (r != kNotHandled) return r;
  }
  return launch_search_simt(ctx, q, nq, db, N, k, scores, ids, ws, st);
}

}  // namespace tq
