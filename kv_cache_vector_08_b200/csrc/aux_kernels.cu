// Small CUDA-core kernels around the tensor-core hot path: query preparation for the
// standalone logits (Pi q, S q), the per-query top-k merge of search candidates, and the
// context-split geometry and workspace layout of decode attention.
#include <algorithm>
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"

namespace tq {

namespace {

template <typename T>
__device__ __forceinline__ float load_f(const T* p);
template <>
__device__ __forceinline__ float load_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// (score, id) ordering of search results: higher score first, equal scores by lower id
__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// ----------------------------------------------------------------------- query prepare
// out[a] = (Pi q_a, S q_a) in fp32.  CTA = 16 queries x 16 outputs (the outputs index the
// concatenation [Pi q | S q]); the terms j run in chunks of 128: the chunk's 16 columns of
// Pi^T / S^T and the 16 query rows are staged in shared memory with one round of loads,
// thread (query, 4 outputs, quarter of the chunk) accumulates 4 dot products, and the
// quarters (adjacent lanes) are summed by shuffles at the end.
constexpr int kPqRows = 16, kPqCols = 16, kPqChunk = 128;

template <typename T>
__global__ void __launch_bounds__(256) prepare_queries_kernel(const T* __restrict__ q, int64_t nq, int64_t ld, int d,
                                                              int m, const float* __restrict__ PiT,
                                                              const float* __restrict__ ST, float* __restrict__ out,
                                                              int64_t out_ld) {
  __shared__ float ms[kPqChunk][kPqCols + 1];
  __shared__ float xs[kPqRows][kPqChunk + 1];
  const int64_t r0 = (int64_t)blockIdx.x * kPqRows;
  const int o0 = blockIdx.y * kPqCols;
  const int t = threadIdx.x;
  const int kq = t & 3, og = (t >> 2) & 3, r = t >> 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < d; k0 += kPqChunk) {
    const int kn = min(kPqChunk, d - k0);
    for (int e = t; e < kPqChunk * kPqCols; e += 256) {
      const int jj = e / kPqCols, oc = e % kPqCols, oo = o0 + oc;
      float v = 0.f;
      if (jj < kn) {
        if (oo < d) v = __ldg(PiT + (size_t)(k0 + jj) * d + oo);
        else if (oo < d + m) v = __ldg(ST + (size_t)(k0 + jj) * m + (oo - d));
      }
      ms[jj][oc] = v;
    }
    for (int e = t; e < kPqRows * kPqChunk; e += 256) {
      const int rr = e / kPqChunk, jj = e % kPqChunk;
      xs[rr][jj] = (r0 + rr < nq && jj < kn) ? load_f(q + (r0 + rr) * ld + k0 + jj) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = kq; jj < kn; jj += 4) {
      const float x = xs[r][jj];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(ms[jj][4 * og + i], x, acc[i]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 1);
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 2);
  }
  if (kq == 0 && r0 + r < nq)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int oo = o0 + 4 * og + i;
      if (oo < d + m) out[(r0 + r) * out_ld + oo] = acc[i];
    }
}

// One CTA per query: k rounds of arg-max over all candidates.
__global__ void __launch_bounds__(256) search_merge_kernel(float* __restrict__ cand_s,
                                                           int64_t* __restrict__ cand_i, int64_t ncand,
                                                           int k, float* __restrict__ scores,
                                                           int64_t* __restrict__ ids) {
  const int64_t a = blockIdx.x;
  float* s = cand_s + a * ncand;
  int64_t* ix = cand_i + a * ncand;
  __shared__ float ws[8];
  __shared__ int64_t wi[8];
  __shared__ int64_t wpos[8];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int64_t bi = INT64_MAX, bp = -1;
    for (int64_t j = threadIdx.x; j < ncand; j += blockDim.x)
      if (better(s[j], ix[j], bs, bi)) { bs = s[j]; bi = ix[j]; bp = j; }
    for (int o = 16; o > 0; o >>= 1) {
      float os = __shfl_xor_sync(0xffffffffu, bs, o);
      int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      int64_t op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (better(os, oi, bs, bi)) { bs = os; bi = oi; bp = op; }
    }
    if (lane == 0) { ws[warp] = bs; wi[warp] = bi; wpos[warp] = bp; }
    __syncthreads();
    if (threadIdx.x == 0) {
      float fs = ws[0];
      int64_t fi = wi[0], fp = wpos[0];
      for (int w = 1; w < (int)(blockDim.x / 32); ++w)
        if (better(ws[w], wi[w], fs, fi)) { fs = ws[w]; fi = wi[w]; fp = wpos[w]; }
      scores[a * k + r] = fs;
      ids[a * k + r] = fi;
      if (fp >= 0) { s[fp] = -INFINITY; ix[fp] = INT64_MAX; }
    }
    __syncthreads();
  }
}

}  // namespace

int launch_prepare_queries(const tq_ctx* ctx, const void* q, int q_dtype, int64_t nq, int64_t ld, float* out,
                           int64_t out_ld, cudaStream_t st) {
  if (nq == 0) return TQ_OK;
  int d = ctx->lay.d, m = ctx->m;
  dim3 grid((unsigned)div_up(nq, kPqRows), (unsigned)div_up(d + m, kPqCols));
  if (q_dtype == TQ_DTYPE_F32)
    prepare_queries_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), nq, ld, d, m, ctx->PiT, ctx->ST,
                                                        out, out_ld);
  else if (q_dtype == TQ_DTYPE_BF16)
    prepare_queries_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), nq, ld, d, m,
                                                                ctx->PiT, ctx->ST, out, out_ld);
  else
    return fail(TQ_ERR_INVALID_ARG, "query dtype must be TQ_DTYPE_F32 or TQ_DTYPE_BF16");
  count_launch();
  return check_launch("prepare_queries_kernel");
}

// Resident decode CTAs on the current device: its SM count times the CTAs per SM the
// tensor-core decode kernel is built for (registers bound it); 148 SMs when no device can
// be queried.
static int decode_slots() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  return decode_mma_ctas_per_sm() * sms;
}

// Context splits per (sequence, kv head): each CTA streams `chunk` tokens (a multiple of
// the 64-token stage).  The split count minimises the modelled time
//   waves(s) * (tiles per CTA + 2),   waves(s) = ceil(B Hkv s / slots),
// i.e. whole waves of equal CTAs plus a per-CTA start-up of about two stages, so that a
// grid slightly larger than one wave (B Hkv = 512 on 444 slots) is split into several
// nearly full waves instead of leaving a second, almost empty one.
void decode_geometry(int B, int Hkv, int64_t max_len, int* nsplit, int* chunk) {
  constexpr int64_t kTile = 64;
  int64_t tiles = (max_len + kTile - 1) / kTile;
  if (tiles < 1) tiles = 1;
  const int64_t bh = (int64_t)B * Hkv > 0 ? (int64_t)B * Hkv : 1;
  const int64_t slots = decode_slots();
  int64_t best_s = 1;
  double best_t = 1e300;
  const int64_t smax = std::min<int64_t>(512, tiles);
  for (int64_t s = 1; s <= smax; ++s) {
    const int64_t per = (tiles + s - 1) / s;
    if (s > 1 && (tiles + per - 1) / per < s) continue;     // same split as a smaller s
    const int64_t waves = (bh * s + slots - 1) / slots;
    const double t = (double)waves * (double)(per + 2);
    if (t < best_t - 1e-9) {
      best_t = t;
      best_s = s;
    }
  }
  const int64_t tiles_per = (tiles + best_s - 1) / best_s;
  *chunk = (int)(tiles_per * kTile);
  *nsplit = (int)((tiles + tiles_per - 1) / tiles_per);
}

// Workspace: prepared queries [B*Hq][G][2*D], split partials [B*Hq][nsplit][D+2], each
// region 256-byte aligned.
DecodeWs decode_ws(int B, int Hq, int Hkv, int D, int G, int64_t max_len) {
  DecodeWs w{};
  const int nsub = Hkv > 0 ? (Hq / Hkv + 3) / 4 : 1;      // CTAs per (sequence, kv head): 4 query heads each
  decode_geometry(B, Hkv * nsub, max_len, &w.nsplit, &w.chunk);
  auto up = [](size_t x) { return ((x + 255) / 256) * 256; };
  w.qp = 0;
  w.part = up((size_t)B * Hq * G * 2 * D * sizeof(float));
  w.part_ld = ((int64_t)w.nsplit * (D + 2) + 3) / 4 * 4;
  w.total = w.part + up((size_t)B * Hq * w.part_ld * sizeof(float));
  return w;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int ngroups, int64_t max_len, int) {
  return decode_ws(B, Hq, Hkv, D, ngroups, max_len).total;
}

int launch_search_merge(float* cand_s, int64_t* cand_i, int64_t nq, int64_t ncand, int k, float* scores, int64_t* ids,
                        cudaStream_t st) {
  search_merge_kernel<<<(unsigned)nq, 256, 0, st>>>(cand_s, cand_i, ncand, k, scores, ids);
  count_launch();
  return check_launch("search_merge_kernel");
}

}  // namespace tq
