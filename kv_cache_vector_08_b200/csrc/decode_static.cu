// Decode attention for callers that cannot allocate device memory: the split-K scratch
// (prepared queries and per-split partial softmax states) lives in a fixed-size array in
// this library's own device memory instead of a caller-provided workspace.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace tq {
namespace {

// The scratch array.  Every GPU that loads this library's device code holds it until the
// process exits.  Host code must never pass `g_decode_scratch` itself to a kernel: on the
// host that name is only a stand-in for the symbol, not a device address.  The device
// address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[TQ_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; looked up on the first call
// for each device (with that device current) and cached for the life of the process.  A
// cudaDeviceReset of that device invalidates the cached address.
int static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TQ_ERR_UNSUPPORTED, "device ordinal above 127");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" int tq_decode_attention_static(const tq_ctx* const* kctx, const tq_ctx* const* vctx,
                                          const int* group_off, int ngroups, const void* q, int q_dtype,
                                          const tq_packed* kcache, const tq_packed* vcache,
                                          const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                                          int64_t max_len, float scale, float* out, tq_stream_t stream) {
  // the arguments first (an invalid shape is TQ_ERR_INVALID_ARG whatever its size), then the
  // scratch size, then the array's address; nothing is launched before all three pass
  int r = tq::check_decode_args(kctx, vctx, group_off, ngroups, q, q_dtype, kcache, vcache, seq_lens, B, Hq, Hkv, D,
                                max_len, out, 0);
  if (r != TQ_OK) return r;
  if (B == 0) return TQ_OK;
  size_t need = tq_decode_workspace_size(B, Hq, Hkv, D, ngroups, max_len);
  if (need > (size_t)TQ_DECODE_STATIC_SCRATCH_BYTES)
    return tq::fail(TQ_ERR_WORKSPACE,
                    "tq_decode_attention_static: this shape needs " + std::to_string(need) +
                        " bytes of scratch but the static scratch holds " +
                        std::to_string((size_t)TQ_DECODE_STATIC_SCRATCH_BYTES) +
                        " bytes; use tq_decode_attention with a caller workspace");
  void* scratch = nullptr;
  r = tq::static_scratch(&scratch);
  if (r != TQ_OK) return r;
  // Nothing in the scratch has to start at zero: the query-preparation kernel writes every
  // prepared query and the split kernel writes every partial state before the merge reads it.
  return tq_decode_attention(kctx, vctx, group_off, ngroups, q, q_dtype, kcache, vcache, seq_lens, B, Hq, Hkv, D,
                             max_len, scale, out, scratch, (size_t)TQ_DECODE_STATIC_SCRATCH_BYTES, stream);
}
