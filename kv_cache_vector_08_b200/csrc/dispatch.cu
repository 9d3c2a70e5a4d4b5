// Kernel-family selection for each hot-path call.
#include "common.cuh"
#include "kernels.cuh"


namespace tq {

int launch_quantize(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                    const int64_t* slots, void* ws, size_t ws_bytes, cudaStream_t st) {
  // the fused bf16 kernel where it applies, the workspace path (any shape) otherwise
  int r = launch_quantize_tc(ctx, x, x_dtype, n, ld, dst, slots, st);
  if (r != kNotHandled) return r;
  return launch_quantize_gen(ctx, x, x_dtype, n, ld, nullptr, dst, slots, ws, ws_bytes, st);
}

int launch_logits(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* logits,
                  void* ws, cudaStream_t st) {
  int r = launch_logits_mma(ctx, q, nq, keys, n, logits, ws, st);
  if (r != kNotHandled) return r;
  return fail(TQ_ERR_UNSUPPORTED,
              "tq_attn_logits: supported for prod-mode contexts with d in {64, 128} and 2-4 code bits, keys 16-byte "
              "aligned");
}

int launch_decode(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G, const int32_t* perm,
                  const int32_t* table, int page, const void* q, int q_dtype, const tq_packed* kc,
                  const tq_packed* vc, const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len,
                  float scale, float* out, void* ws, cudaStream_t st) {
  int r = launch_decode_mma(kctx, vctx, off, G, perm, table, page, q, q_dtype, kc, vc, seq_lens, B, Hq, Hkv, D,
                            max_len, scale, out, ws, st);
  if (r != kNotHandled) return r;
  return fail(TQ_ERR_UNSUPPORTED,
              "tq_decode_attention: supported channel groups are one group of d = 128 with 4 + 4 or 3 + 3 key / value "
              "bits, or two groups of d = 64 with (4 + 4, 3 + 3) or (3 + 3, 2 + 2) bits; caches and norms 16-byte "
              "aligned; at most 512 context splits");
}

int launch_search(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                  float* scores, int64_t* ids, void* ws, cudaStream_t st) {
  return launch_search_tc(ctx, q, nq, db, N, k, scores, ids, ws, st);
}

}  // namespace tq
