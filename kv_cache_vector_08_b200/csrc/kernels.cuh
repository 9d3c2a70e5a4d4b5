// Launchers of the libtq kernels (host side).
#pragma once

#include "common.cuh"

namespace tq {

// Returned by a kernel family's launcher when it does not cover the requested shape.
constexpr int kNotHandled = -1;

int launch_prepare_queries(const tq_ctx* ctx, const void* q, int q_dtype, int64_t nq, int64_t ld, float* out,
                           int64_t out_ld, cudaStream_t st);
void decode_geometry(int B, int Hkv, int64_t max_len, int* nsplit, int* chunk);
int decode_mma_ctas_per_sm();
struct DecodeWs {
  size_t qp, part, total;       // byte offsets of the regions and total size
  int nsplit, chunk;
  int64_t part_ld;              // floats per query row of the split partials (16-byte multiple)
};
DecodeWs decode_ws(int B, int Hq, int Hkv, int D, int G, int64_t max_len);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int ngroups, int64_t max_len, int qp_ld);
int launch_dequantize_tc(const tq_ctx* ctx, const tq_packed* src, const int64_t* slots, int64_t n, float* out,
                         int64_t ld, bool qjl, cudaStream_t st);
size_t quantize_gen_workspace(const tq_ctx* ctx, int64_t n);
int launch_quantize_gen(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const int32_t* cols,
                        const tq_packed* dst, const int64_t* slots, void* ws, size_t ws_bytes, cudaStream_t st);
bool quantize_tc_applies(const tq_ctx* ctx, int x_dtype, int64_t n, int64_t ld);
int launch_quantize_tc(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                       const int64_t* slots, cudaStream_t st);
int launch_decode_mma(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G,
                      const int32_t* perm, const int32_t* table, int page, const void* q, int q_dtype,
                      const tq_packed* kc, const tq_packed* vc, const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                      int64_t max_len, float scale, float* out, void* ws, cudaStream_t st);
size_t logits_mma_workspace(int64_t nq, int d);
int launch_logits_mma(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* out,
                      void* ws, cudaStream_t st);
size_t search_tc_workspace(const tq_ctx* ctx, int64_t nq, int64_t N, int k);
int launch_search_tc(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                     float* scores, int64_t* ids, void* ws, cudaStream_t st);
int launch_search_merge(float* cand_s, int64_t* cand_i, int64_t nq, int64_t ncand, int k, float* scores, int64_t* ids,
                        cudaStream_t st);

}  // namespace tq

namespace tq {
// Dispatchers: pick the fastest kernel family that supports the shape.
int launch_quantize(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                    const int64_t* slots, void* ws, size_t ws_bytes, cudaStream_t st);
int launch_logits(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* logits,
                  void* ws, cudaStream_t st);
int launch_decode(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G, const int32_t* perm,
                  const int32_t* table, int page, const void* q, int q_dtype, const tq_packed* kc,
                  const tq_packed* vc, const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len,
                  float scale, float* out, void* ws, cudaStream_t st);
int check_decode_args(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* group_off, int ngroups,
                      const void* q, int q_dtype, const tq_packed* kcache, const tq_packed* vcache,
                      const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int64_t max_len, const float* out,
                      int page);
int launch_search(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                  float* scores, int64_t* ids, void* ws, cudaStream_t st);
}  // namespace tq
