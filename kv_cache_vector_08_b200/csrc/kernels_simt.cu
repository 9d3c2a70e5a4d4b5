// SIMT (CUDA-core) kernels of the TurboQuant hot path: quantize, dequantize, query
// preparation, attention logits, split-K decode attention + merge, search scan + top-k.
// They accept every supported (d, bits, mode) and are the reference rung for the
// tensor-core kernels, which take over the shapes of the KV-cache workloads.
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
template <>
__device__ __forceinline__ float load_f<__half>(const __half* p) { return __half2float(*p); }

__device__ __forceinline__ double warp_sum_d(double v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sumf(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint16_t f16_bits(float v) { return __half_as_ushort(__float2half_rn(v)); }

// index of the nearest centroid: number of boundaries strictly below y
__device__ __forceinline__ int nearest(float y, const float* t, int K) {
  int idx = 0;
  for (int j = 0; j < K - 1; ++j) idx += (y > t[j]) ? 1 : 0;
  return idx;
}

// The P-bit code of coordinate i of a record (index code in bits 0..k-1, the QJL sign
// in bit k in prod mode).
__device__ __forceinline__ uint32_t read_code(const uint8_t* rec, const Layout& L, int i) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(rec) + (i >> 5) * L.planes;
  uint32_t c = 0;
  for (int b = 0; b < L.planes; ++b) {
    const int q = code_bit_pos(L.planes, i & 31, b);
    c |= ((w[q >> 5] >> (q & 31)) & 1u) << b;
  }
  return c;
}

// The P words of group g of a record, into registers (P <= 5).
__device__ __forceinline__ void load_group(const uint8_t* rec, const Layout& L, int g, uint32_t (&w)[5]) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(rec) + g * L.planes;
  for (int b = 0; b < L.planes; ++b) w[b] = src[b];
}

// ---------------------------------------------------------------------------- quantize
// One CTA quantizes VT vectors: norm, y = Pi x / ||x||, nearest centroid, residual
// r = y - c[idx], ||r||, signs of M r (M = S Pi^T), then packs the planes.
template <typename T, int VT, bool PROD>
__global__ void __launch_bounds__(128) quantize_simt_kernel(
    const T* __restrict__ x, int64_t n, int64_t ld, const float* __restrict__ PiT,
    const float* __restrict__ MT, Codebook cb, Layout L, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ norm, uint16_t* __restrict__ rnorm, const int64_t* __restrict__ slots) {
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  const int d = L.d, dp = L.d_pad;
  float* xs = smem;                 // [VT][dp] input, fp32
  float* ys = xs + VT * dp;         // [VT][dp] y, then r
  float* nrm = ys + VT * dp;        // [VT]
  float* rn = nrm + VT;             // [VT]
  float* ct = rn + VT;              // [16] centroids, [16] boundaries
  uint8_t* ids = reinterpret_cast<uint8_t*>(ct + 32);  // [VT][dp]
  uint8_t* sg = ids + VT * dp;                          // [VT][dp]
  const int64_t v0 = (int64_t)blockIdx.x * VT;
  const int nv = (int)min((int64_t)VT, n - v0);
  if (threadIdx.x < 16) {
    ct[threadIdx.x] = cb.c[threadIdx.x];
    ct[16 + threadIdx.x] = cb.t[threadIdx.x];
  }
  for (int e = threadIdx.x; e < VT * dp; e += blockDim.x) {
    int v = e / dp, i = e % dp;
    xs[e] = (v < nv && i < d) ? load_f(x + (v0 + v) * ld + i) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  for (int v = warp; v < VT; v += nw) {
    double s = 0.0;
    for (int i = lane; i < d; i += 32) s += (double)xs[v * dp + i] * xs[v * dp + i];
    s = warp_sum_d(s);
    if (lane == 0) nrm[v] = (float)sqrt(s);
  }
  __syncthreads();
  // y_i = sum_j Pi[i][j] x_j / ||x||   (PiT[j][i] = Pi[i][j]: coalesced over i)
  for (int i = threadIdx.x; i < dp; i += blockDim.x) {
    float acc[VT];
#pragma unroll
    for (int v = 0; v < VT; ++v) acc[v] = 0.f;
    if (i < d) {
      for (int j = 0; j < d; ++j) {
        float p = PiT[(size_t)j * d + i];
#pragma unroll
        for (int v = 0; v < VT; ++v) acc[v] = fmaf(p, xs[v * dp + j], acc[v]);
      }
    }
#pragma unroll
    for (int v = 0; v < VT; ++v) {
      float nv_ = nrm[v];
      float y = (nv_ > 0.f) ? acc[v] / nv_ : 0.f;
      int idx = nearest(y, ct + 16, cb.K);
      ids[v * dp + i] = (uint8_t)((i < d) ? idx : 0);
      ys[v * dp + i] = (i < d) ? (y - ct[idx]) : 0.f;
    }
  }
  __syncthreads();
  if (PROD) {
    for (int v = warp; v < VT; v += nw) {
      double s = 0.0;
      for (int i = lane; i < d; i += 32) s += (double)ys[v * dp + i] * ys[v * dp + i];
      s = warp_sum_d(s);
      if (lane == 0) rn[v] = (float)sqrt(s);
    }
    // z_j = sum_i M[j][i] r_i, sign bit = [z_j >= 0]
    for (int j = threadIdx.x; j < dp; j += blockDim.x) {
      float acc[VT];
#pragma unroll
      for (int v = 0; v < VT; ++v) acc[v] = 0.f;
      if (j < d) {
        for (int i = 0; i < d; ++i) {
          float mm = MT[(size_t)i * d + j];
#pragma unroll
          for (int v = 0; v < VT; ++v) acc[v] = fmaf(mm, ys[v * dp + i], acc[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < VT; ++v)
        sg[v * dp + j] = (j < d) ? ((acc[v] >= 0.f || nrm[v] == 0.f) ? 1 : 0) : 0;
    }
  }
  __syncthreads();
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    int64_t slot = slots ? slots[v0 + v] : v0 + v;
    bool zero = nrm[v] == 0.f;
    norm[slot] = f16_bits(nrm[v]);
    if (PROD) rnorm[slot] = zero ? (uint16_t)0 : f16_bits(rn[v]);
  }
  // pack: one thread per output word (every code bit has one place in its group's words)
  const int P = L.planes, nwords = L.code_bytes / 4;
  for (int e = threadIdx.x; e < nv * nwords; e += blockDim.x) {
    const int v = e / nwords, W = e % nwords, g = W / P, wi = W % P;
    uint32_t word = 0;
    for (int c = 0; c < 32; ++c) {
      const int i = g * 32 + c;
      if (i >= d) break;
      const uint32_t code = index_code(ids[v * dp + i], L.k) | ((uint32_t)sg[v * dp + i] << L.k);
      for (int b = 0; b < P; ++b) {
        const int q = code_bit_pos(P, c, b);
        if ((q >> 5) == wi) word |= ((code >> b) & 1u) << (q & 31);
      }
    }
    int64_t slot = slots ? slots[v0 + v] : v0 + v;
    reinterpret_cast<uint32_t*>(codes + slot * L.code_bytes)[W] = word;
  }
}

template <typename T, int VT>
int launch_quantize_t(const tq_ctx* ctx, const void* x, int64_t n, int64_t ld, const tq_packed* dst,
                      const int64_t* slots, cudaStream_t st) {
  const Layout& L = ctx->lay;
  size_t smem = (size_t)VT * L.d_pad * (2 * sizeof(float) + 2) + (2 * VT + 32) * sizeof(float);
  auto kern = ctx->mode == TQ_MODE_PROD ? quantize_simt_kernel<T, VT, true> : quantize_simt_kernel<T, VT, false>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(quantize)");
  }
  int grid = div_up(n, VT);
  kern<<<grid, 128, smem, st>>>(static_cast<const T*>(x), n, ld, ctx->PiT, ctx->MT, ctx->cb, L, dst->codes,
                                dst->norm, dst->rnorm, slots);
  count_launch();
  return check_launch("quantize_simt_kernel");
}

template <typename T>
int launch_quantize_dt(const tq_ctx* ctx, const void* x, int64_t n, int64_t ld, const tq_packed* dst,
                       const int64_t* slots, cudaStream_t st) {
  int dp = ctx->lay.d_pad;
  if (dp <= 256) return launch_quantize_t<T, 16>(ctx, x, n, ld, dst, slots, st);
  if (dp <= 1024) return launch_quantize_t<T, 4>(ctx, x, n, ld, dst, slots, st);
  return launch_quantize_t<T, 1>(ctx, x, n, ld, dst, slots, st);
}

// --------------------------------------------------------------------------- dequantize
template <int VT>
__global__ void __launch_bounds__(128) dequantize_simt_kernel(
    const float* __restrict__ Pi, Codebook cb, Layout L, const uint8_t* __restrict__ codes,
    const uint16_t* __restrict__ norm, const int64_t* __restrict__ slots, int64_t n,
    float* __restrict__ out, int64_t ld) {
  extern __shared__ float4 smem4[];
  float* cv = reinterpret_cast<float*>(smem4);  // [VT][dp] centroid values c[idx_i]
  float* nn = cv + VT * L.d_pad;                // [VT]
  const int d = L.d, dp = L.d_pad;
  const int64_t v0 = (int64_t)blockIdx.x * VT;
  const int nv = (int)min((int64_t)VT, n - v0);
  for (int e = threadIdx.x; e < VT * dp; e += blockDim.x) {
    int v = e / dp, i = e % dp;
    float val = 0.f;
    if (v < nv && i < d) {
      int64_t slot = slots ? slots[v0 + v] : v0 + v;
      val = cb.cc[read_code(codes + slot * L.code_bytes, L, i) & (uint32_t)(cb.K - 1)];
    }
    cv[e] = val;
  }
  if (threadIdx.x < VT) {
    int v = threadIdx.x;
    nn[v] = 0.f;
    if (v < nv) nn[v] = __half2float(__ushort_as_half(norm[slots ? slots[v0 + v] : v0 + v]));
  }
  __syncthreads();
  // x_hat_j = ||x|| sum_i Pi[i][j] c[idx_i]   (Pi row-major: coalesced over j)
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc[VT];
#pragma unroll
    for (int v = 0; v < VT; ++v) acc[v] = 0.f;
    for (int i = 0; i < d; ++i) {
      float p = Pi[(size_t)i * d + j];
#pragma unroll
      for (int v = 0; v < VT; ++v) acc[v] = fmaf(p, cv[v * dp + i], acc[v]);
    }
    for (int v = 0; v < nv; ++v) out[(v0 + v) * ld + j] = nn[v] * acc[v];
  }
}

// ----------------------------------------------------------------------- query prepare
// out[a] = (Pi q_a, S q_a); one thread per output coordinate.
template <typename T>
__global__ void prepare_queries_kernel(const T* __restrict__ q, int64_t nq, int64_t ld, int d, int m,
                                       const float* __restrict__ PiT, const float* __restrict__ ST,
                                       float* __restrict__ out, int64_t out_ld) {
  int64_t a = blockIdx.y;
  int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= nq || o >= d + m) return;
  const T* qa = q + a * ld;
  float acc = 0.f;
  if (o < d) {
    for (int j = 0; j < d; ++j) acc = fmaf(PiT[(size_t)j * d + o], load_f(qa + j), acc);
  } else {
    int r = o - d;
    for (int j = 0; j < d; ++j) acc = fmaf(ST[(size_t)j * m + r], load_f(qa + j), acc);
  }
  out[a * out_ld + o] = acc;
}

// ------------------------------------------------------------------------------ logits
// One thread per key, QT queries per CTA (blockIdx.y selects the query tile).
template <int QT>
__global__ void __launch_bounds__(128) logits_simt_kernel(
    const float* __restrict__ qprep, int64_t nq, int qld, Codebook cb, Layout L, int prod, float coef,
    const uint8_t* __restrict__ codes, const uint16_t* __restrict__ norm,
    const uint16_t* __restrict__ rnorm, int64_t n, float* __restrict__ logits) {
  extern __shared__ float4 smem4[];
  float* qt = reinterpret_cast<float*>(smem4);  // [QT][dp]
  float* qs = qt + QT * L.d_pad;                // [QT][dp]
  float* ct = qs + QT * L.d_pad;                // [16]
  const int d = L.d, dp = L.d_pad;
  const int64_t a0 = (int64_t)blockIdx.y * QT;
  const int na = (int)min((int64_t)QT, nq - a0);
  for (int e = threadIdx.x; e < QT * dp; e += blockDim.x) {
    int a = e / dp, i = e % dp;
    bool ok = a < na && i < d;
    qt[e] = ok ? qprep[(a0 + a) * qld + i] : 0.f;
    qs[e] = (ok && prod) ? qprep[(a0 + a) * qld + d + i] : 0.f;
  }
  if (threadIdx.x < 16) ct[threadIdx.x] = cb.cc[threadIdx.x];
  __syncthreads();
  int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n) return;
  const uint8_t* rec = codes + b * L.code_bytes;
  float mse[QT], qjl[QT];
#pragma unroll
  for (int a = 0; a < QT; ++a) mse[a] = qjl[a] = 0.f;
  const uint32_t kmask = (uint32_t)(cb.K - 1);
  for (int g = 0; g * 32 < d; ++g) {
    uint32_t w[5];
    load_group(rec, L, g, w);
    for (int e = 0; e < 32 && g * 32 + e < d; ++e) {
      const int i = g * 32 + e;
      const uint32_t code = group_code(w, L.planes, e);
      float c = ct[code & kmask];
      bool s = prod ? ((code >> L.k) & 1u) : false;
#pragma unroll
      for (int a = 0; a < QT; ++a) {
        mse[a] = fmaf(qt[a * dp + i], c, mse[a]);
        float v = qs[a * dp + i];
        qjl[a] += s ? v : -v;
      }
    }
  }
  float nk = __half2float(__ushort_as_half(norm[b]));
  float rk = prod ? __half2float(__ushort_as_half(rnorm[b])) : 0.f;
  for (int a = 0; a < na; ++a) logits[(a0 + a) * n + b] = nk * (mse[a] + coef * rk * qjl[a]);
}

// ------------------------------------------------------------------------------ decode
constexpr int kDecTile = 128;  // tokens per tile = threads per CTA
constexpr int kMaxRep = 8;     // query heads per kv head handled by one CTA
constexpr int kMaxGroups = 4;

struct DecodeGroup {
  Codebook kcb, vcb;
  Layout kl, vl;
  float coef;
  int off;
  const uint8_t* kcodes;
  const uint16_t* knorm;
  const uint16_t* krnorm;
  const uint8_t* vcodes;
  const uint16_t* vnorm;
};

struct DecodeArgs {
  DecodeGroup g[kMaxGroups];
  int G, B, Hq, Hkv, D, rep, nsplit, chunk, qp_ld;
  int64_t max_len;
  float scale;
  const int32_t* seq_lens;
  const float* qprep;  // [B*Hq][G][2*qp_ld]: (Pi q, S q) per group
  float* part;         // [B*Hq][nsplit][D+2]
};

// One CTA per (split, b*Hkv + hk): online softmax over the split's tokens for all rep
// query heads; values accumulated in each group's rotated basis.
__global__ void __launch_bounds__(kDecTile) decode_split_simt_kernel(DecodeArgs A) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  const int D = A.D, rep = A.rep, G = A.G;
  float* qt = sm;                        // [rep][D]
  float* qs = qt + rep * D;              // [rep][D]
  float* lg = qs + rep * D;              // [rep][kDecTile] logits, then p
  float* red = lg + rep * kDecTile;      // [rep][4] per-warp partials
  float* vn = red + rep * 4;             // [G][kDecTile] value norms
  float* cvt = vn + G * kDecTile;        // [G][16] value centroids
  float* ckt = cvt + G * 16;             // [G][16] key centroids
  uint8_t* vcs = reinterpret_cast<uint8_t*>(ckt + G * 16);  // [G][kDecTile][vbytes_g]
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / A.Hkv, hk = bh % A.Hkv;
  const int T = max(0, (int)min((int64_t)A.seq_lens[b], A.max_len));
  const int t_begin = split * A.chunk;
  const int t_end = min(T, t_begin + A.chunk);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  for (int e = tid; e < rep * D; e += blockDim.x) {
    int h = e / D, c = e % D;
    int g = 0;
    while (g + 1 < G && c >= A.g[g + 1].off) ++g;
    int i = c - A.g[g].off;
    const float* src = A.qprep + ((size_t)(b * A.Hq + hk * rep + h) * G + g) * 2 * A.qp_ld;
    qt[e] = src[i];
    qs[e] = src[A.g[g].kl.d + i];   // prepared row = (Pi q [d_g], S q [d_g])
  }
  if (tid < 16)
    for (int g = 0; g < G; ++g) {
      cvt[g * 16 + tid] = A.g[g].vcb.cc[tid];
      ckt[g * 16 + tid] = A.g[g].kcb.cc[tid];
    }
  float m_run[kMaxRep], l_run[kMaxRep], acc[kMaxRep][2];
#pragma unroll
  for (int h = 0; h < kMaxRep; ++h) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
    acc[h][0] = acc[h][1] = 0.f;
  }
  __syncthreads();
  const int64_t slot0 = (int64_t)bh * A.max_len;
  for (int ts = t_begin; ts < t_end; ts += kDecTile) {
    const int t = ts + tid;
    const bool valid = t < t_end;
    // phase A: logits of token t for every query head
    float logit[kMaxRep];
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) logit[h] = 0.f;
    if (valid) {
      for (int g = 0; g < G; ++g) {
        const DecodeGroup& gr = A.g[g];
        const Layout& L = gr.kl;
        const uint8_t* rec = gr.kcodes + (slot0 + t) * L.code_bytes;
        float mse[kMaxRep], qjl[kMaxRep];
#pragma unroll
        for (int h = 0; h < kMaxRep; ++h) mse[h] = qjl[h] = 0.f;
        const uint32_t kmask = (uint32_t)(gr.kcb.K - 1);
        for (int gg = 0; gg * 32 < L.d; ++gg) {
          uint32_t w[5];
          load_group(rec, L, gg, w);
          for (int e = 0; e < 32 && gg * 32 + e < L.d; ++e) {
            const uint32_t code = group_code(w, L.planes, e);
            float c = ckt[g * 16 + (code & kmask)];
            bool s = (code >> L.k) & 1u;
            int col = gr.off + gg * 32 + e;
#pragma unroll
            for (int h = 0; h < kMaxRep; ++h) {
              if (h < rep) {
                mse[h] = fmaf(qt[h * D + col], c, mse[h]);
                float v = qs[h * D + col];
                qjl[h] += s ? v : -v;
              }
            }
          }
        }
        float nk = __half2float(__ushort_as_half(gr.knorm[slot0 + t]));
        float rk = __half2float(__ushort_as_half(gr.krnorm[slot0 + t]));
#pragma unroll
        for (int h = 0; h < kMaxRep; ++h) logit[h] += nk * (mse[h] + gr.coef * rk * qjl[h]);
      }
    }
    for (int h = 0; h < rep; ++h) lg[h * kDecTile + tid] = valid ? logit[h] * A.scale : -INFINITY;
    // stage the tile's value codes and norms
    for (int g = 0; g < G; ++g) {
      const DecodeGroup& gr = A.g[g];
      int vb = gr.vl.code_bytes;
      uint8_t* dst = vcs;
      for (int gg = 0; gg < g; ++gg) dst += kDecTile * A.g[gg].vl.code_bytes;
      int ntok = min(kDecTile, t_end - ts);
      const uint8_t* src = gr.vcodes + (slot0 + ts) * vb;
      for (int e = tid; e < ntok * vb; e += blockDim.x) dst[e] = src[e];
      vn[g * kDecTile + tid] = valid ? __half2float(__ushort_as_half(gr.vnorm[slot0 + t])) : 0.f;
    }
    __syncthreads();
    // phase B: tile max and sum per head
    float m_new[kMaxRep], alpha[kMaxRep];
    for (int h = 0; h < rep; ++h) {
      float v = warp_max(lg[h * kDecTile + tid]);
      if (lane == 0) red[h * 4 + warp] = v;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      if (h < rep) {
        float tm = fmaxf(fmaxf(red[h * 4 + 0], red[h * 4 + 1]), fmaxf(red[h * 4 + 2], red[h * 4 + 3]));
        m_new[h] = fmaxf(m_run[h], tm);
        alpha[h] = __expf(m_run[h] - m_new[h]);
      }
    }
    __syncthreads();
    for (int h = 0; h < rep; ++h) {
      float p = valid ? __expf(lg[h * kDecTile + tid] - m_new[h]) : 0.f;
      lg[h * kDecTile + tid] = p;
      float s = warp_sumf(p);
      if (lane == 0) red[h * 4 + warp] = s;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      if (h < rep) {
        l_run[h] = l_run[h] * alpha[h] + (red[h * 4] + red[h * 4 + 1] + red[h * 4 + 2] + red[h * 4 + 3]);
        m_run[h] = m_new[h];
        acc[h][0] *= alpha[h];
        acc[h][1] *= alpha[h];
      }
    }
    // phase C: value accumulation, thread <-> channel (tid, tid + kDecTile)
    const int ntok = min(kDecTile, t_end - ts);
    for (int cc = 0; cc < 2; ++cc) {
      int col = tid + cc * kDecTile;
      if (col >= D) break;
      int g = 0;
      while (g + 1 < G && col >= A.g[g + 1].off) ++g;
      const DecodeGroup& gr = A.g[g];
      const Layout& L = gr.vl;
      const uint8_t* tile = vcs;
      for (int gg = 0; gg < g; ++gg) tile += kDecTile * A.g[gg].vl.code_bytes;
      const int i = col - gr.off;
      const uint32_t vmask = (uint32_t)(gr.vcb.K - 1);
      for (int tt = 0; tt < ntok; ++tt) {
        const uint8_t* rec = tile + tt * L.code_bytes;
        const uint32_t code = read_code(rec, L, i);
        float cv = cvt[g * 16 + (code & vmask)] * vn[g * kDecTile + tt];
#pragma unroll
        for (int h = 0; h < kMaxRep; ++h)
          if (h < rep) acc[h][cc] = fmaf(lg[h * kDecTile + tt], cv, acc[h][cc]);
      }
    }
    __syncthreads();
  }
  // partial results: (m, l, acc) per query head
  for (int h = 0; h < rep; ++h) {
    float* dst = A.part + ((size_t)(b * A.Hq + hk * rep + h) * A.nsplit + split) * (D + 2);
    if (tid == 0) {
      dst[0] = m_run[h];
      dst[1] = l_run[h];
    }
    for (int cc = 0; cc < 2; ++cc) {
      int col = tid + cc * kDecTile;
      if (col < D) dst[2 + col] = acc[h][cc];
    }
  }
}

struct MergeArgs {
  const float* part;
  int nsplit, D, G;
  int off[kMaxGroups + 1];
  const float* PiV[kMaxGroups];  // value rotations [d_g][d_g]
  float* out;
};

// One CTA per (b, h): log-sum-exp merge of the splits, then o = Pi_v^T acc per group.
__global__ void __launch_bounds__(128) decode_merge_kernel(MergeArgs A) {
  extern __shared__ float4 smem4[];
  float* accr = reinterpret_cast<float*>(smem4);  // [D]
  float* w = accr + A.D;                          // [nsplit]
  const int bh = blockIdx.x, D = A.D;
  const float* P = A.part + (size_t)bh * A.nsplit * (D + 2);
  __shared__ float sL;
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int s = 0; s < A.nsplit; ++s) M = fmaxf(M, P[(size_t)s * (D + 2)]);
    float L = 0.f;
    for (int s = 0; s < A.nsplit; ++s) {
      float ms = P[(size_t)s * (D + 2)];
      float ws = (ms == -INFINITY) ? 0.f : __expf(ms - M);
      w[s] = ws;
      L += ws * P[(size_t)s * (D + 2) + 1];
    }
    sL = L;
  }
  __syncthreads();
  const float invL = sL > 0.f ? 1.f / sL : 0.f;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < A.nsplit; ++s) a = fmaf(w[s], P[(size_t)s * (D + 2) + 2 + c], a);
    accr[c] = a * invL;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    int g = 0;
    while (g + 1 < A.G && c >= A.off[g + 1]) ++g;
    int lo = A.off[g], dg = A.off[g + 1] - lo, j = c - lo;
    const float* Pi = A.PiV[g];
    float o = 0.f;
    for (int i = 0; i < dg; ++i) o = fmaf(Pi[(size_t)i * dg + j], accr[lo + i], o);
    A.out[(size_t)bh * D + c] = o;
  }
}

// ------------------------------------------------------------------------------ search
constexpr int kSearchBlock = 1024;  // database vectors per CTA
constexpr int kSearchQT = 4;        // queries per CTA

__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Scores of kSearchQT queries against kSearchBlock database vectors, then the block's
// top-k of each query into the candidate buffer.
__global__ void __launch_bounds__(256) search_block_kernel(
    const float* __restrict__ qprep, int64_t nq, int qld, Codebook cb, Layout L, float coef,
    const uint8_t* __restrict__ codes, const uint16_t* __restrict__ norm,
    const uint16_t* __restrict__ rnorm, int64_t N, int k, float* __restrict__ cand_s,
    int64_t* __restrict__ cand_i) {
  extern __shared__ float4 smem4[];
  float* qt = reinterpret_cast<float*>(smem4);  // [QT][dp]
  float* qs = qt + kSearchQT * L.d_pad;         // [QT][dp]
  float* sc = qs + kSearchQT * L.d_pad;         // [QT][block]
  float* ct = sc + kSearchQT * kSearchBlock;    // [16]
  const int d = L.d, dp = L.d_pad;
  const int64_t a0 = (int64_t)blockIdx.y * kSearchQT;
  const int na = (int)min((int64_t)kSearchQT, nq - a0);
  const int64_t n0 = (int64_t)blockIdx.x * kSearchBlock;
  for (int e = threadIdx.x; e < kSearchQT * dp; e += blockDim.x) {
    int a = e / dp, i = e % dp;
    bool ok = a < na && i < d;
    qt[e] = ok ? qprep[(a0 + a) * qld + i] : 0.f;
    qs[e] = ok ? qprep[(a0 + a) * qld + d + i] : 0.f;
  }
  if (threadIdx.x < 16) ct[threadIdx.x] = cb.cc[threadIdx.x];
  __syncthreads();
  for (int r = threadIdx.x; r < kSearchBlock; r += blockDim.x) {
    int64_t b = n0 + r;
    float mse[kSearchQT], qjl[kSearchQT];
#pragma unroll
    for (int a = 0; a < kSearchQT; ++a) mse[a] = qjl[a] = 0.f;
    if (b < N) {
      const uint8_t* rec = codes + b * L.code_bytes;
      const uint32_t kmask = (uint32_t)(cb.K - 1);
      for (int g = 0; g * 32 < d; ++g) {
        uint32_t w[5];
        load_group(rec, L, g, w);
        for (int e = 0; e < 32 && g * 32 + e < d; ++e) {
          const int i = g * 32 + e;
          const uint32_t code = group_code(w, L.planes, e);
          float c = ct[code & kmask];
          bool s = (code >> L.k) & 1u;
#pragma unroll
          for (int a = 0; a < kSearchQT; ++a) {
            mse[a] = fmaf(qt[a * dp + i], c, mse[a]);
            float v = qs[a * dp + i];
            qjl[a] += s ? v : -v;
          }
        }
      }
      float nk = __half2float(__ushort_as_half(norm[b]));
      float rk = __half2float(__ushort_as_half(rnorm[b]));
#pragma unroll
      for (int a = 0; a < kSearchQT; ++a) sc[a * kSearchBlock + r] = nk * (mse[a] + coef * rk * qjl[a]);
    } else {
#pragma unroll
      for (int a = 0; a < kSearchQT; ++a) sc[a * kSearchBlock + r] = -INFINITY;
    }
  }
  __syncthreads();
  // per query (one warp each): k rounds of arg-max with (score desc, id asc)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nblk = gridDim.x;
  if (warp < na) {
    float* s = sc + warp * kSearchBlock;
    for (int r = 0; r < k; ++r) {
      float bs = -INFINITY;
      int bi = kSearchBlock;
      for (int j = lane; j < kSearchBlock; j += 32)
        if (s[j] > bs || (s[j] == bs && j < bi)) { bs = s[j]; bi = j; }
      for (int o = 16; o > 0; o >>= 1) {
        float os = __shfl_xor_sync(0xffffffffu, bs, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (os > bs || (os == bs && oi < bi)) { bs = os; bi = oi; }
      }
      size_t at = ((size_t)(a0 + warp) * nblk + blockIdx.x) * k + r;
      if (lane == 0) {
        bool ok = bi < kSearchBlock && n0 + bi < N && bs != -INFINITY;
        cand_s[at] = ok ? bs : -INFINITY;
        cand_i[at] = ok ? n0 + bi : INT64_MAX;
        if (bi < kSearchBlock) s[bi] = -INFINITY;
      }
      __syncwarp();
    }
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

// ============================================================================ launchers
int launch_quantize_simt(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld,
                         const tq_packed* dst, const int64_t* slots, cudaStream_t st) {
  if (n == 0) return TQ_OK;
  switch (x_dtype) {
    case TQ_DTYPE_F32: return launch_quantize_dt<float>(ctx, x, n, ld, dst, slots, st);
    case TQ_DTYPE_BF16: return launch_quantize_dt<__nv_bfloat16>(ctx, x, n, ld, dst, slots, st);
    case TQ_DTYPE_F16: return launch_quantize_dt<__half>(ctx, x, n, ld, dst, slots, st);
  }
  return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_DTYPE_F32, BF16 or F16");
}

int launch_dequantize_simt(const tq_ctx* ctx, const tq_packed* src, const int64_t* slots, int64_t n,
                           float* out, int64_t ld, cudaStream_t st) {
  if (n == 0) return TQ_OK;
  constexpr int VT = 8;
  size_t smem = (size_t)VT * ctx->lay.d_pad * sizeof(float) + VT * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(dequantize_simt_kernel<VT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(dequantize)");
  }
  dequantize_simt_kernel<VT><<<div_up(n, VT), 128, smem, st>>>(ctx->Pi, ctx->cb, ctx->lay, src->codes, src->norm,
                                                               slots, n, out, ld);
  count_launch();
  return check_launch("dequantize_simt_kernel");
}

int launch_prepare_queries(const tq_ctx* ctx, const void* q, int q_dtype, int64_t nq, int64_t ld, float* out,
                           int64_t out_ld, cudaStream_t st) {
  if (nq == 0) return TQ_OK;
  int d = ctx->lay.d, m = ctx->m;
  dim3 grid(div_up(d + m, 128), (unsigned)nq);
  if (q_dtype == TQ_DTYPE_F32)
    prepare_queries_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float*>(q), nq, ld, d, m, ctx->PiT, ctx->ST,
                                                        out, out_ld);
  else if (q_dtype == TQ_DTYPE_BF16)
    prepare_queries_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q), nq, ld, d, m,
                                                                ctx->PiT, ctx->ST, out, out_ld);
  else
    return fail(TQ_ERR_INVALID_ARG, "query dtype must be TQ_DTYPE_F32 or TQ_DTYPE_BF16");
  count_launch();
  return check_launch("prepare_queries_kernel");
}

int launch_logits_simt(const tq_ctx* ctx, const float* qprep, int64_t nq, const tq_packed* keys, int64_t n,
                       float* logits, cudaStream_t st) {
  if (nq == 0 || n == 0) return TQ_OK;
  constexpr int QT = 8;
  size_t smem = (size_t)2 * QT * ctx->lay.d_pad * sizeof(float) + 16 * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(logits_simt_kernel<QT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(logits)");
  }
  dim3 grid(div_up(n, 128), div_up(nq, QT));
  logits_simt_kernel<QT><<<grid, 128, smem, st>>>(qprep, nq, ctx->lay.d + ctx->m, ctx->cb, ctx->lay,
                                                  ctx->mode == TQ_MODE_PROD, ctx->sqrt_pi_over_2_over_m, keys->codes,
                                                  keys->norm, keys->rnorm, n, logits);
  count_launch();
  return check_launch("logits_simt_kernel");
}

// split-K geometry shared by the size query and every decode launch: the context is cut
// into chunks of whole 64-token tiles so that about 3 CTAs per SM are in flight.
void decode_geometry(int B, int Hkv, int64_t max_len, int* nsplit, int* chunk) {
  constexpr int64_t kTile = 64;
  int64_t tiles = (max_len + kTile - 1) / kTile;
  if (tiles < 1) tiles = 1;
  int64_t bh = (int64_t)B * Hkv;
  int64_t want = (3 * 148 + bh - 1) / bh;   // one wave at 3 CTAs per SM
  if (want < 1) want = 1;
  if (want > 512) want = 512;
  if (want > tiles) want = tiles;
  int64_t tiles_per = (tiles + want - 1) / want;
  *chunk = (int)(tiles_per * kTile);
  *nsplit = (int)((tiles + tiles_per - 1) / tiles_per);
}

// Workspace: prepared queries [B*Hq][G][2*D], split partials [B*Hq][nsplit][D+2],
// completion counters [B*Hkv] (each region 256-byte aligned).
DecodeWs decode_ws(int B, int Hq, int Hkv, int D, int G, int64_t max_len) {
  DecodeWs w{};
  decode_geometry(B, Hkv, max_len, &w.nsplit, &w.chunk);
  auto up = [](size_t x) { return ((x + 255) / 256) * 256; };
  w.qp = 0;
  w.part = up((size_t)B * Hq * G * 2 * D * sizeof(float));
  w.part_ld = ((int64_t)w.nsplit * (D + 2) + 3) / 4 * 4;
  w.cnt = w.part + up((size_t)B * Hq * w.part_ld * sizeof(float));
  w.total = w.cnt + up((size_t)B * Hkv * sizeof(int));
  return w;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int ngroups, int64_t max_len, int) {
  return decode_ws(B, Hq, Hkv, D, ngroups, max_len).total;
}

int launch_decode_simt(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G, const void* q,
                       int q_dtype, const tq_packed* kc, const tq_packed* vc, const int32_t* seq_lens, int B, int Hq,
                       int Hkv, int D, int64_t max_len, float scale, float* out, void* ws, cudaStream_t st) {
  if (G > kMaxGroups) return fail(TQ_ERR_UNSUPPORTED, "at most 4 channel groups");
  const int rep = Hq / Hkv;
  if (rep > kMaxRep) return fail(TQ_ERR_UNSUPPORTED, "at most 8 query heads per kv head");
  if (D > 2 * kDecTile) return fail(TQ_ERR_UNSUPPORTED, "head dimension above 256");
  const int qp_ld = D;
  const DecodeWs W = decode_ws(B, Hq, Hkv, D, G, max_len);
  const int nsplit = W.nsplit, chunk = W.chunk;
  float* qprep = reinterpret_cast<float*>(static_cast<char*>(ws) + W.qp);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + W.part);
  // query preparation per group: rows (b, h) of q restricted to the group's channels
  for (int g = 0; g < G; ++g) {
    int esz = q_dtype == TQ_DTYPE_F32 ? 4 : 2;
    const char* qg = static_cast<const char*>(q) + (size_t)off[g] * esz;
    int r = launch_prepare_queries(kctx[g], qg, q_dtype, (int64_t)B * Hq, D, qprep + (size_t)g * 2 * qp_ld,
                                   (int64_t)G * 2 * qp_ld, st);
    if (r != TQ_OK) return r;
  }
  DecodeArgs A{};
  A.G = G; A.B = B; A.Hq = Hq; A.Hkv = Hkv; A.D = D; A.rep = rep;
  A.nsplit = nsplit; A.chunk = chunk; A.qp_ld = qp_ld; A.max_len = max_len; A.scale = scale;
  A.seq_lens = seq_lens; A.qprep = qprep; A.part = part;
  size_t vbytes = 0;
  for (int g = 0; g < G; ++g) {
    DecodeGroup& gr = A.g[g];
    gr.kcb = kctx[g]->cb; gr.vcb = vctx[g]->cb;
    gr.kl = kctx[g]->lay; gr.vl = vctx[g]->lay;
    gr.coef = kctx[g]->sqrt_pi_over_2_over_m;
    gr.off = off[g];
    gr.kcodes = kc[g].codes; gr.knorm = kc[g].norm; gr.krnorm = kc[g].rnorm;
    gr.vcodes = vc[g].codes; gr.vnorm = vc[g].norm;
    vbytes += (size_t)kDecTile * vctx[g]->lay.code_bytes;
  }
  size_t smem = (size_t)(2 * rep * D + rep * kDecTile + rep * 4 + G * kDecTile + 32 * G) * sizeof(float) + vbytes;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  }
  dim3 grid(nsplit, B * Hkv);
  decode_split_simt_kernel<<<grid, kDecTile, smem, st>>>(A);
  count_launch();
  int r = check_launch("decode_split_simt_kernel");
  if (r != TQ_OK) return r;
  return launch_decode_merge(vctx, off, G, part, nsplit, B * Hq, D, out, st);
}

int launch_decode_merge(const tq_ctx* const* vctx, const int* off, int G, const float* part, int nsplit, int BHq,
                        int D, float* out, cudaStream_t st) {
  MergeArgs M{};
  M.part = part; M.nsplit = nsplit; M.D = D; M.G = G; M.out = out;
  for (int g = 0; g < G; ++g) { M.off[g] = off[g]; M.PiV[g] = vctx[g]->Pi; }
  M.off[G] = D;
  decode_merge_kernel<<<BHq, 128, (D + nsplit) * sizeof(float), st>>>(M);
  count_launch();
  return check_launch("decode_merge_kernel");
}

size_t search_workspace_bytes(const tq_ctx* ctx, int64_t nq, int64_t N, int k) {
  int64_t nblk = (N + kSearchBlock - 1) / kSearchBlock;
  size_t qp = (size_t)nq * (ctx->lay.d + ctx->m) * sizeof(float);
  size_t cand = (size_t)nq * nblk * k;
  return ((qp + 255) / 256) * 256 + ((cand * sizeof(float) + 255) / 256) * 256 + cand * sizeof(int64_t);
}

int launch_search_simt(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                       float* scores, int64_t* ids, void* ws, cudaStream_t st) {
  if (nq == 0) return TQ_OK;
  int64_t nblk = (N + kSearchBlock - 1) / kSearchBlock;
  int qld = ctx->lay.d + ctx->m;
  size_t qp = (size_t)nq * qld * sizeof(float);
  size_t cand = (size_t)nq * nblk * k;
  float* qprep = static_cast<float*>(ws);
  char* p = static_cast<char*>(ws) + ((qp + 255) / 256) * 256;
  float* cs = reinterpret_cast<float*>(p);
  int64_t* ci = reinterpret_cast<int64_t*>(p + ((cand * sizeof(float) + 255) / 256) * 256);
  int r = launch_prepare_queries(ctx, q, TQ_DTYPE_F32, nq, ctx->lay.d, qprep, qld, st);
  if (r != TQ_OK) return r;
  size_t smem = ((size_t)2 * kSearchQT * ctx->lay.d_pad + kSearchQT * kSearchBlock + 16) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(search_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(search)");
  }
  dim3 grid((unsigned)nblk, div_up(nq, kSearchQT));
  search_block_kernel<<<grid, 256, smem, st>>>(qprep, nq, qld, ctx->cb, ctx->lay, ctx->sqrt_pi_over_2_over_m,
                                               db->codes, db->norm, db->rnorm, N, k, cs, ci);
  count_launch();
  r = check_launch("search_block_kernel");
  if (r != TQ_OK) return r;
  return launch_search_merge(cs, ci, nq, nblk * k, k, scores, ids, st);
}

int launch_search_merge(float* cand_s, int64_t* cand_i, int64_t nq, int64_t ncand, int k, float* scores, int64_t* ids,
                        cudaStream_t st) {
  search_merge_kernel<<<(unsigned)nq, 256, 0, st>>>(cand_s, cand_i, ncand, k, scores, ids);
  count_launch();
  return check_launch("search_merge_kernel");
}

}  // namespace tq
