// Top-k search over a packed database on the tensor cores (int8 mma.sync).
//
// turboquant.net "核心用例 · 向量搜索": the database is the quantized key set, every query is
// scored by the unbiased inner-product estimator
//   score(q, k) = ||k|| (<Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, sign(S r)>),
// and the top-k by score are returned (ties by lower id).  Scoring is a dense contraction
// [keys x d] x [d x queries], run as the decode kernel's key path: centroids as two int8
// digits of a 16-bit fixed point (A operand, decoded from the packed words with byte
// permutes), the prepared queries as two int8 digits in the 8 MMA columns (4 queries x
// hi/lo), QJL signs as sign-replicated bytes.  The database is 4-bit prod codes (3-bit
// index + sign), any d (padded to 32).
//
// Layout of the work: CTA = (group of 16 queries, range of 1024 keys), 4 warps.  Each warp
// scores 16-key tiles; for every 32-coordinate block it decodes the A fragments once and
// applies them to the 4 query blocks of the group (12 MMAs).  Consecutive CTAs share the
// key range (the query group varies fastest), so a range is read from HBM once and from L2
// by the other groups.  Scores go to shared memory; each warp then extracts the top-k of
// 4 queries by k rounds of warp arg-max and writes them as candidates of the range; the
// candidates of all ranges are merged per query by the search merge kernel.
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_ops.cuh"

namespace tq {
namespace {

using namespace mmaops;

constexpr int kQG = 16;         // queries per CTA (4 blocks of 4)
constexpr int kRange = 1024;    // keys per CTA
constexpr int kMaxK = 32;       // largest k of this kernel

// Per-query fixed point of the prepared query (Pi q, S q): int16 [nq][2][d_pad] scaled by
// 32000 / max |.| of each part, the scale inverses and the sum of the S q part.
__global__ void __launch_bounds__(128) search_fixq_kernel(const float* __restrict__ qprep, int d, int d_pad, int nq,
                                                          int16_t* __restrict__ qfix, float* __restrict__ qsc) {
  const int a = blockIdx.x;
  __shared__ float red[2][4];
  __shared__ int ired[4];
  const float* src = qprep + (size_t)a * 2 * d;
  float mx[2] = {0.f, 0.f};
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    mx[0] = fmaxf(mx[0], fabsf(src[i]));
    mx[1] = fmaxf(mx[1], fabsf(src[d + i]));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int p = 0; p < 2; ++p) {
    float v = mx[p];
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[p][warp] = v;
  }
  __syncthreads();
  float scale[2];
  for (int p = 0; p < 2; ++p) {
    const float m = fmaxf(fmaxf(red[p][0], red[p][1]), fmaxf(red[p][2], red[p][3]));
    scale[p] = m > 0.f ? kFix / m : 0.f;
    if (threadIdx.x == 0) qsc[a * 3 + p] = m / kFix;
  }
  int ssum = 0;
  for (int i = threadIdx.x; i < d_pad; i += blockDim.x) {
    const int v0 = i < d ? __float2int_rn(src[i] * scale[0]) : 0;
    const int v1 = i < d ? __float2int_rn(src[d + i] * scale[1]) : 0;
    qfix[((size_t)a * 2 + 0) * d_pad + i] = (int16_t)v0;
    qfix[((size_t)a * 2 + 1) * d_pad + i] = (int16_t)v1;
    ssum += v1;
  }
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
  if (lane == 0) ired[warp] = ssum;
  __syncthreads();
  if (threadIdx.x == 0) qsc[a * 3 + 2] = (float)(ired[0] + ired[1] + ired[2] + ired[3]);
}

// B fragments [query group][block][query block][lane]: (digits of Pi q for k-slots 4l..4l+3,
// for 16+4l..16+4l+3, then the same for S q); lane (g, l) = column g (query 4 qb + g/2,
// hi digit for g even, lo for g odd), coordinates 32 b + 8 l + j.
__global__ void __launch_bounds__(128) search_frag_kernel(const int16_t* __restrict__ qfix, int d_pad, int nq,
                                                          uint4* __restrict__ frag) {
  const int qg = blockIdx.x, b = blockIdx.y, nblk = gridDim.y;
  const int qb = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  const int a = qg * kQG + qb * 4 + (g >> 1);
  const bool lo = (g & 1) != 0;
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (a < nq) {
    for (int part = 0; part < 2; ++part) {
      const int16_t* q = qfix + ((size_t)a * 2 + part) * d_pad + 32 * b + 8 * l;
      for (int h = 0; h < 2; ++h) {
        uint32_t v = 0;
        for (int t = 0; t < 4; ++t) {
          const int x = q[4 * h + t];
          const int hi = (x + 128) >> 8;
          v |= (uint32_t)(uint8_t)(lo ? x - (hi << 8) : hi) << (8 * t);
        }
        w[part * 2 + h] = v;
      }
    }
  }
  frag[(((size_t)qg * nblk + b) * 4 + qb) * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
}

struct SearchArgs {
  const uint8_t* codes;
  const uint16_t* norm;
  const uint16_t* rnorm;
  const uint4* frag;      // [nqg][nblk][4][32]
  const float* qsc;       // [nq][3]: 1/s_m, 1/s_s, sum of S q digits
  int64_t N;
  int nq, nblk, code_bytes, k;
  uint32_t kh[2], kl[2];  // key centroid digits by code
  float coef, kc_inv;
  float* cand_s;          // [nq][nrange][k]
  int64_t* cand_i;
  int64_t nrange;
};

__device__ __forceinline__ float h2f(unsigned short h) { return __half2float(__ushort_as_half(h)); }

__global__ void __launch_bounds__(128) search_mma_kernel(SearchArgs A) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint4* s_frag = reinterpret_cast<uint4*>(sm);                                   // [nblk][4][32]
  float* s_sc = reinterpret_cast<float*>(sm + (size_t)A.nblk * 4 * 32 * 16);     // [16][kRange]
  const int qg = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * kRange;
  const int64_t r1 = min(A.N, r0 + kRange);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, l = lane & 3;
  for (int i = threadIdx.x; i < A.nblk * 4 * 32; i += blockDim.x)
    s_frag[i] = A.frag[(size_t)qg * A.nblk * 4 * 32 + i];
  // per-query constants of this thread's 4 queries (column head l of every query block)
  float inv_m[4], inv_s[4], sum_s[4];
#pragma unroll
  for (int qb = 0; qb < 4; ++qb) {
    const int a = qg * kQG + qb * 4 + l;
    const bool ok = a < A.nq;
    inv_m[qb] = ok ? A.qsc[a * 3 + 0] : 0.f;
    inv_s[qb] = ok ? A.qsc[a * 3 + 1] : 0.f;
    sum_s[qb] = ok ? A.qsc[a * 3 + 2] : 0.f;
  }
  __syncthreads();
  const int cb = A.code_bytes;
  for (int t0 = warp * 16; t0 < kRange; t0 += 64) {
    const int64_t ka = r0 + t0 + g, kb = ka + 8;
    const bool va = ka < r1, vb = kb < r1;
    int acc[4][3][4];
#pragma unroll
    for (int qb = 0; qb < 4; ++qb)
#pragma unroll
      for (int j = 0; j < 3; ++j) acc[qb][j][0] = acc[qb][j][1] = acc[qb][j][2] = acc[qb][j][3] = 0;
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(A.codes + (va ? ka : 0) * cb) + l;
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(A.codes + (vb ? kb : 0) * cb) + l;
    uint32_t na = va ? __ldg(pa) : 0u, nb = vb ? __ldg(pb) : 0u;
    for (int b = 0; b < A.nblk; ++b) {
      const uint32_t wa = na, wb = nb;
      if (b + 1 < A.nblk) {
        na = va ? __ldg(pa + 4 * (b + 1)) : 0u;
        nb = vb ? __ldg(pb + 4 * (b + 1)) : 0u;
      }
      // slice l of block b: low 3 code bits as nibbles, top (sign) bits at byte msbs
      const uint32_t sa = wa & 0x77777777u, sb = wb & 0x77777777u;
      const uint32_t sa1 = sa >> 16, sb1 = sb >> 16;
      const uint32_t h0 = prmt(A.kh[0], A.kh[1], sa), h1 = prmt(A.kh[0], A.kh[1], sb);
      const uint32_t h2 = prmt(A.kh[0], A.kh[1], sa1), h3 = prmt(A.kh[0], A.kh[1], sb1);
      const uint32_t l0 = prmt(A.kl[0], A.kl[1], sa), l1 = prmt(A.kl[0], A.kl[1], sb);
      const uint32_t l2 = prmt(A.kl[0], A.kl[1], sa1), l3 = prmt(A.kl[0], A.kl[1], sb1);
      const uint32_t s0 = msb_bytes(wa), s1 = msb_bytes(wb), s2 = msb_bytes(wa << 4), s3 = msb_bytes(wb << 4);
#pragma unroll
      for (int qb = 0; qb < 4; ++qb) {
        const uint4 f = s_frag[(b * 4 + qb) * 32 + lane];
        mma_s8(acc[qb][0], h0, h1, h2, h3, f.x, f.y);
        mma_s8(acc[qb][1], l0, l1, l2, l3, f.x, f.y);
        mma_s8(acc[qb][2], s0, s1, s2, s3, f.z, f.w);
      }
    }
    const float nka = va ? h2f(__ldg(A.norm + ka)) : 0.f, rka = va ? h2f(__ldg(A.rnorm + ka)) : 0.f;
    const float nkb = vb ? h2f(__ldg(A.norm + kb)) : 0.f, rkb = vb ? h2f(__ldg(A.rnorm + kb)) : 0.f;
#pragma unroll
    for (int qb = 0; qb < 4; ++qb) {
      // columns 2l (query hi digit), 2l+1 (lo digit); rows g (i = 0) and g+8 (i = 2)
      auto score = [&](int i, float n, float r) {
        const float mse = fmaf(65536.f, (float)acc[qb][0][i],
                               fmaf(256.f, (float)acc[qb][0][i + 1] + (float)acc[qb][1][i], (float)acc[qb][1][i + 1]));
        const float sq = fmaf(-2.f, fmaf(256.f, (float)acc[qb][2][i], (float)acc[qb][2][i + 1]), -sum_s[qb]);
        return n * fmaf(A.coef * r, sq * inv_s[qb], mse * A.kc_inv * inv_m[qb]);
      };
      float* row = s_sc + (qb * 4 + l) * kRange;
      row[t0 + g] = va ? score(0, nka, rka) : -INFINITY;
      row[t0 + g + 8] = vb ? score(2, nkb, rkb) : -INFINITY;
    }
  }
  __syncthreads();
  // top-k of queries 4 warp .. 4 warp + 3 of the group: k rounds of warp arg-max
  for (int qq = 0; qq < 4; ++qq) {
    const int qi = warp * 4 + qq;
    const int a = qg * kQG + qi;
    float* row = s_sc + qi * kRange;
    for (int r = 0; r < A.k; ++r) {
      float bs = -INFINITY;
      int bj = kRange;
      for (int j = lane; j < kRange; j += 32)
        if (row[j] > bs) { bs = row[j]; bj = j; }   // ascending j: first maximum per lane
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (os > bs || (os == bs && oj < bj)) { bs = os; bj = oj; }
      }
      if (lane == 0 && a < A.nq) {
        const size_t c = ((size_t)a * A.nrange + blockIdx.y) * A.k + r;
        A.cand_s[c] = bs;
        A.cand_i[c] = (bs == -INFINITY) ? INT64_MAX : r0 + bj;
      }
      if (lane == (bj & 31) && bj < kRange) row[bj] = -INFINITY;
      __syncwarp();
    }
  }
}

}  // namespace

size_t search_mma_workspace(const tq_ctx* ctx, int64_t nq, int64_t N, int k) {
  const int d = ctx->lay.d, d_pad = ctx->lay.d_pad, nblk = d_pad / 32;
  const int64_t nqg = (nq + kQG - 1) / kQG, nrange = (N + kRange - 1) / kRange;
  auto up = [](size_t x) { return ((x + 255) / 256) * 256; };
  return up((size_t)nq * 2 * d * 4) + up((size_t)nq * 2 * d_pad * 2) + up((size_t)nq * 3 * 4) +
         up((size_t)nqg * nblk * 4 * 32 * 16) + up((size_t)nq * nrange * k * 4) + (size_t)nq * nrange * k * 8;
}

// 4-bit prod databases with k <= 32; kNotHandled otherwise.
int launch_search_mma(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                      float* scores, int64_t* ids, void* ws, cudaStream_t st) {
  if (ctx->mode != TQ_MODE_PROD || ctx->lay.planes != 4 || k > kMaxK || k < 1) return kNotHandled;
  if ((reinterpret_cast<uintptr_t>(db->codes) & 15) != 0) return kNotHandled;
  const int d = ctx->lay.d, d_pad = ctx->lay.d_pad, nblk = d_pad / 32;
  const int64_t nqg = (nq + kQG - 1) / kQG, nrange = (N + kRange - 1) / kRange;
  if (nqg > 65535 || nrange > 65535) return kNotHandled;
  const size_t smem = (size_t)nblk * 4 * 32 * 16 + (size_t)kQG * kRange * 4;
  if (smem > 200 * 1024) return kNotHandled;
  auto up = [](size_t x) { return ((x + 255) / 256) * 256; };
  char* p = static_cast<char*>(ws);
  float* qprep = reinterpret_cast<float*>(p);
  p += up((size_t)nq * 2 * d * 4);
  int16_t* qfix = reinterpret_cast<int16_t*>(p);
  p += up((size_t)nq * 2 * d_pad * 2);
  float* qsc = reinterpret_cast<float*>(p);
  p += up((size_t)nq * 3 * 4);
  uint4* frag = reinterpret_cast<uint4*>(p);
  p += up((size_t)nqg * nblk * 4 * 32 * 16);
  float* cs = reinterpret_cast<float*>(p);
  p += up((size_t)nq * nrange * k * 4);
  int64_t* ci = reinterpret_cast<int64_t*>(p);
  int r = launch_prepare_queries(ctx, q, TQ_DTYPE_F32, nq, d, qprep, 2 * d, st);
  if (r != TQ_OK) return r;
  search_fixq_kernel<<<(unsigned)nq, 128, 0, st>>>(qprep, d, d_pad, (int)nq, qfix, qsc);
  count_launch();
  if ((r = check_launch("search_fixq_kernel")) != TQ_OK) return r;
  search_frag_kernel<<<dim3((unsigned)nqg, (unsigned)nblk), 128, 0, st>>>(qfix, d_pad, (int)nq, frag);
  count_launch();
  if ((r = check_launch("search_frag_kernel")) != TQ_OK) return r;
  SearchArgs A{};
  A.codes = db->codes; A.norm = db->norm; A.rnorm = db->rnorm; A.frag = frag; A.qsc = qsc;
  A.N = N; A.nq = (int)nq; A.nblk = nblk; A.code_bytes = ctx->lay.code_bytes; A.k = k;
  Luts t;
  A.kc_inv = host_luts(ctx, ctx, &t);
  A.kh[0] = t.kh[0]; A.kh[1] = t.kh[1]; A.kl[0] = t.kl[0]; A.kl[1] = t.kl[1];
  A.coef = ctx->sqrt_pi_over_2_over_m;
  A.cand_s = cs; A.cand_i = ci; A.nrange = nrange;
  cudaError_t e = cudaFuncSetAttribute(search_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(search_mma_kernel)");
  search_mma_kernel<<<dim3((unsigned)nqg, (unsigned)nrange), 128, smem, st>>>(A);
  count_launch();
  if ((r = check_launch("search_mma_kernel")) != TQ_OK) return r;
  return launch_search_merge(cs, ci, nq, nrange * k, k, scores, ids, st);
}

}  // namespace tq
