// Decode attention over the packed cache on the tensor cores, operands built in registers.
//
// turboquant.net "集成到 Attention": keys and values stay quantized and attention reads
// them directly; admirer.cn (H100 paragraph): the attention-logit computation on 4-bit
// keys is where the speed-up is measured.  Per cached token and GQA group of query heads
// the work is a small dense contraction (4 heads x 128 coordinates for the MSE term, the
// QJL sign term and the value accumulation), so each warp runs it on mma.sync m16n8k16:
//
//   logits^T [16 tokens x 8] = Ck [16 x 16k] * [q~_hi | q~_lo]      (MSE term, 4 heads)
//                            + Sk [16 x 16k] * [q^_hi | q^_lo]      (QJL term, +-1 signs)
//   out^T   [16 coords x 8]  += Cv^T [16 x 16 tokens] * [P_hi | P_lo]
//
// The A operands are produced straight from the packed bit planes in registers: the
// bit planes of four coordinates form a prmt selector that looks the fp16 centroid
// bytes up in register-resident tables (4 lookups per prmt); signs become +-1.0 with one
// shift and one LOP3 per pair; the value tile is turned around with movmatrix.  The hi/lo
// halves of the queries and of the probabilities ride in the 8 columns of each MMA, so the
// fp16 rounding of the queries and probabilities costs no extra MMA.  Centroids are used
// at fp16 precision (relative error <= 2^-11), well inside the output tolerance.
//
// One CTA (4 warps) handles one (sequence, kv head, context split); warps take 16-token
// tiles in turn, keep an online softmax (log2 domain) per head, and merge their states in
// shared memory before writing one partial (m, l, acc) per query head and split.
#include <cfloat>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace tq {
namespace {

constexpr int kWarps = 4;
constexpr int kRep = 4;   // query heads per kv head handled by this kernel

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movT(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Static description of one channel group handled by the kernel.
template <int DG_, int KK_, int KV_>
struct GroupCfg {
  static constexpr int DG = DG_;            // group width (64 or 128)
  static constexpr int Q = DG_ / 4;         // coordinates per quarter
  static constexpr int KK = KK_;            // key index bits (prod mode)
  static constexpr int KV = KV_;            // value index bits (MSE mode)
  static constexpr int PK = KK_ + 1;        // key planes
  static constexpr int PV = KV_;            // value planes
  static constexpr int NKB = DG_ / 16;      // 16-coordinate k-blocks
  static constexpr uint32_t M1 = (Q == 32) ? 0x11111111u : 0x1111u;
};

// Quarter l of one record: planes as 32-bit words (16 valid bits when Q = 16).
template <int Q, int P>
__device__ __forceinline__ void load_quarter(const uint8_t* rec, int l, uint32_t (&w)[P]) {
  if constexpr (Q == 32) {
    const uint8_t* p = rec + l * (4 * P);
    if constexpr (P == 4) {
      uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (P == 2) {
      uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
    }
  } else {
    const uint8_t* p = rec + l * (2 * P);
    if constexpr (P == 4) {
      uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = v.x & 0xFFFFu; w[1] = v.x >> 16; w[2] = v.y & 0xFFFFu; w[3] = v.y >> 16;
    } else if constexpr (P == 2) {
      uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p));
      w[0] = v & 0xFFFFu; w[1] = v >> 16;
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) w[i] = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    }
  }
}

// prmt selector nibbles (3 index bits) for coordinates 4k + qq of a quarter.
template <int NB, uint32_t M1>
__device__ __forceinline__ uint32_t selector(const uint32_t* w, int qq) {
  uint32_t s = (w[0] >> qq) & M1;
  if constexpr (NB > 1) s |= ((w[1] >> qq) & M1) << 1;
  if constexpr (NB > 2) s |= ((w[2] >> qq) & M1) << 2;
  return s;
}

// fp16 centroid table split into low/high bytes, 8 entries per register pair.
struct Lut {
  uint32_t lo[4], hi[4];  // lo[0..1]: low bytes of c[0..7], lo[2..3]: of c[8..15]
};

__device__ __forceinline__ Lut make_lut(const float* c, int K) {
  Lut t;
  uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
  for (int j = 0; j < 16; ++j) {
    uint16_t b = j < K ? __half_as_ushort(__float2half_rn(c[j])) : 0;
    lo[j / 4] |= (uint32_t)(b & 0xFF) << (8 * (j % 4));
    hi[j / 4] |= (uint32_t)(b >> 8) << (8 * (j % 4));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) { t.lo[i] = lo[i]; t.hi[i] = hi[i]; }
  return t;
}

// Two half2 registers: fp16 centroids of the coordinates selected by the 4 nibbles of
// `sel` (pairs nibble 0,1 and nibble 2,3).  NB index bits; the 4th bit (NB == 4) chooses
// between the two 8-entry tables through `sel4` (nibble k = k + 4*b3_k).
template <int NB>
__device__ __forceinline__ void lookup(const Lut& t, uint32_t sel, uint32_t sel4, uint32_t& x01, uint32_t& x23) {
  uint32_t L, H;
  if constexpr (NB <= 3) {
    L = __byte_perm(t.lo[0], t.lo[1], sel);
    H = __byte_perm(t.hi[0], t.hi[1], sel);
  } else {
    uint32_t La = __byte_perm(t.lo[0], t.lo[1], sel), Lb = __byte_perm(t.lo[2], t.lo[3], sel);
    uint32_t Ha = __byte_perm(t.hi[0], t.hi[1], sel), Hb = __byte_perm(t.hi[2], t.hi[3], sel);
    L = __byte_perm(La, Lb, sel4);
    H = __byte_perm(Ha, Hb, sel4);
  }
  x01 = __byte_perm(L, H, 0x5140);
  x23 = __byte_perm(L, H, 0x7362);
}

// Per-group kernel arguments.
struct MmaGroup {
  const uint8_t* kcodes;
  const uint16_t* knorm;
  const uint16_t* krnorm;
  const uint8_t* vcodes;
  const uint16_t* vnorm;
  float kc[16], vc[16];
  float coef;          // sqrt(pi/2)/m
  int off;             // first channel of the group
  int kbytes, vbytes;  // record sizes
};

struct MmaArgs {
  MmaGroup g[2];
  int B, Hq, Hkv, D, nsplit, chunk, qp_ld, G;
  int64_t max_len;
  float scale_log2;    // softmax scale * log2(e)
  const int32_t* seq_lens;
  const float* qprep;  // [B*Hq][G][2*qp_ld]
  float* part;         // [B*Hq][nsplit][D+2]
};

// Query fragments of one group for this thread, built once per CTA.
template <class GC>
struct QFrag {
  uint32_t mse[GC::NKB][2];
  uint32_t sgn[GC::NKB][2];
};

template <class GC>
__device__ __forceinline__ void load_qfrag(QFrag<GC>& f, const MmaArgs& A, int gi, int b, int hk, int lane) {
  const int g = lane >> 2, l = lane & 3;
  const int head = hk * kRep + (g & 3);
  const bool lo_part = g >= 4;
  const float* src = A.qprep + ((size_t)(b * A.Hq + head) * A.G + gi) * 2 * A.qp_ld;
  const float* qt = src;
  const float* qs = src + GC::DG;
  auto part = [&](float v) {
    float h = __half2float(__float2half_rn(v));
    return lo_part ? v - h : v;
  };
#pragma unroll
  for (int kb = 0; kb < GC::NKB; ++kb) {
    const int qq = kb & 3, hh = kb >> 2;
    const int base = GC::Q * l + qq + 16 * hh;
    f.mse[kb][0] = pack_h2(part(qt[base]), part(qt[base + 4]));
    f.mse[kb][1] = pack_h2(part(qt[base + 8]), part(qt[base + 12]));
    const int sb = GC::Q * l + 2 * kb;
    f.sgn[kb][0] = pack_h2(part(qs[sb]), part(qs[sb + GC::Q / 2]));
    f.sgn[kb][1] = pack_h2(part(qs[sb + 1]), part(qs[sb + 1 + GC::Q / 2]));
  }
}

// MSE + QJL logits of one group for tokens (g, g+8) of a tile, columns 2l, 2l+1.
template <class GC>
__device__ __forceinline__ void group_logits(const QFrag<GC>& qf, const Lut& kl, const uint32_t (&w0)[GC::PK],
                                             const uint32_t (&w1)[GC::PK], float (&mse)[4], float (&sgn)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) mse[i] = sgn[i] = 0.f;
  uint32_t nw0 = ~w0[GC::KK], nw1 = ~w1[GC::KK];
  if constexpr (GC::Q == 16) {
    nw0 = (nw0 & 0xFFu) | ((nw0 & 0xFF00u) << 8);
    nw1 = (nw1 & 0xFFu) | ((nw1 & 0xFF00u) << 8);
  }
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const uint32_t s0 = selector<GC::KK, GC::M1>(w0, qq), s1 = selector<GC::KK, GC::M1>(w1, qq);
#pragma unroll
    for (int hh = 0; hh < GC::DG / 64; ++hh) {
      const int kb = qq + 4 * hh;
      uint32_t a0, a2, a1, a3;
      lookup<GC::KK>(kl, s0 >> (16 * hh), 0, a0, a2);
      lookup<GC::KK>(kl, s1 >> (16 * hh), 0, a1, a3);
      mma16816(mse, a0, a1, a2, a3, qf.mse[kb][0], qf.mse[kb][1]);
    }
  }
#pragma unroll
  for (int kb = 0; kb < GC::NKB; ++kb) {
    const int j0 = 2 * kb;
    uint32_t a0 = ((nw0 << (15 - j0)) & 0x80008000u) | 0x3C003C00u;
    uint32_t a2 = ((nw0 << (14 - j0)) & 0x80008000u) | 0x3C003C00u;
    uint32_t a1 = ((nw1 << (15 - j0)) & 0x80008000u) | 0x3C003C00u;
    uint32_t a3 = ((nw1 << (14 - j0)) & 0x80008000u) | 0x3C003C00u;
    mma16816(sgn, a0, a1, a2, a3, qf.sgn[kb][0], qf.sgn[kb][1]);
  }
}

// Value accumulation of one group: acc[mb] (rows: coordinates, cols: [P_hi | P_lo] heads).
template <class GC>
__device__ __forceinline__ void group_values(const Lut& vl, const uint32_t (&w0)[GC::PV], const uint32_t (&w1)[GC::PV],
                                             uint32_t pb0, uint32_t pb1, float (&acc)[GC::NKB][4]) {
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const uint32_t s0 = selector<(GC::KV < 3 ? GC::KV : 3), GC::M1>(w0, qq);
    const uint32_t s1 = selector<(GC::KV < 3 ? GC::KV : 3), GC::M1>(w1, qq);
    uint32_t b40 = 0, b41 = 0;
    if constexpr (GC::KV == 4) {
      b40 = ((w0[3] >> qq) & GC::M1) << 2;
      b41 = ((w1[3] >> qq) & GC::M1) << 2;
    }
#pragma unroll
    for (int hh = 0; hh < GC::DG / 64; ++hh) {
      const int mb = qq + 4 * hh;
      uint32_t x0f, x0s, x1f, x1s;  // token g / g+8, coordinate blocks f = 0 (first) and 1 (second)
      lookup<GC::KV>(vl, s0 >> (16 * hh), ((b40 >> (16 * hh)) & 0xFFFFu) | 0x3210u, x0f, x0s);
      lookup<GC::KV>(vl, s1 >> (16 * hh), ((b41 >> (16 * hh)) & 0xFFFFu) | 0x3210u, x1f, x1s);
      // rows (coordinates) g: block f = 0, g+8: block f = 1; k (tokens) 2l.. from token g block, 2l+8.. from g+8
      mma16816(acc[mb], movT(x0f), movT(x0s), movT(x1f), movT(x1s), pb0, pb1);
    }
  }
}

template <class G0, class G1>
__global__ void __launch_bounds__(kWarps * 32) decode_mma_kernel(MmaArgs A) {
  constexpr bool TWO = !std::is_same<G1, void>::value;
  using G1c = typename std::conditional<TWO, G1, G0>::type;
  __shared__ float s_m[kWarps][kRep], s_l[kWarps][kRep];
  __shared__ float s_acc[kWarps][kRep][256];
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / A.Hkv, hk = bh % A.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int T = max(0, (int)min((int64_t)A.seq_lens[b], A.max_len));
  const int t_begin = split * A.chunk;
  const int t_end = min(T, t_begin + A.chunk);
  const int64_t slot0 = (int64_t)bh * A.max_len;

  QFrag<G0> qf0;
  load_qfrag<G0>(qf0, A, 0, b, hk, lane);
  QFrag<G1c> qf1;
  if constexpr (TWO) load_qfrag<G1c>(qf1, A, 1, b, hk, lane);
  const Lut kl0 = make_lut(A.g[0].kc, 1 << G0::KK), vl0 = make_lut(A.g[0].vc, 1 << G0::KV);
  Lut kl1, vl1;
  if constexpr (TWO) {
    kl1 = make_lut(A.g[1].kc, 1 << G1c::KK);
    vl1 = make_lut(A.g[1].vc, 1 << G1c::KV);
  }
  float acc0[G0::NKB][4];
  float acc1[G1c::NKB][4];
#pragma unroll
  for (int i = 0; i < G0::NKB; ++i) acc0[i][0] = acc0[i][1] = acc0[i][2] = acc0[i][3] = 0.f;
#pragma unroll
  for (int i = 0; i < G1c::NKB; ++i) acc1[i][0] = acc1[i][1] = acc1[i][2] = acc1[i][3] = 0.f;
  // softmax state for heads h0 = 2(l&1), h0+1 (log2 domain); l_run is this thread's partial sum
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const bool hi_cols = l < 2;

  for (int ts = t_begin + warp * 16; ts < t_end; ts += kWarps * 16) {
    const int ta = ts + g, tb = ts + g + 8;
    const bool va = ta < t_end, vb = tb < t_end;
    const int64_t sa = slot0 + min(ta, T - 1), sb = slot0 + min(tb, T - 1);
    float logit_a[2] = {0.f, 0.f}, logit_b[2] = {0.f, 0.f};
    uint32_t vw0a[G0::PV], vw0b[G0::PV];
    uint32_t vw1a[G1c::PV], vw1b[G1c::PV];
    float nva0, nvb0, nva1 = 0.f, nvb1 = 0.f;
    {
      const MmaGroup& gr = A.g[0];
      uint32_t ka[G0::PK], kb_[G0::PK];
      load_quarter<G0::Q, G0::PK>(gr.kcodes + sa * gr.kbytes, l, ka);
      load_quarter<G0::Q, G0::PK>(gr.kcodes + sb * gr.kbytes, l, kb_);
      load_quarter<G0::Q, G0::PV>(gr.vcodes + sa * gr.vbytes, l, vw0a);
      load_quarter<G0::Q, G0::PV>(gr.vcodes + sb * gr.vbytes, l, vw0b);
      const float nka = __half2float(__ushort_as_half(__ldg(gr.knorm + sa)));
      const float nkb = __half2float(__ushort_as_half(__ldg(gr.knorm + sb)));
      const float rka = __half2float(__ushort_as_half(__ldg(gr.krnorm + sa)));
      const float rkb = __half2float(__ushort_as_half(__ldg(gr.krnorm + sb)));
      nva0 = __half2float(__ushort_as_half(__ldg(gr.vnorm + sa)));
      nvb0 = __half2float(__ushort_as_half(__ldg(gr.vnorm + sb)));
      float mse[4], sgn[4];
      group_logits<G0>(qf0, kl0, ka, kb_, mse, sgn);
      // columns 2l, 2l+1: add the hi/lo halves held by lanes l and l^2
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mse[i] += __shfl_xor_sync(0xffffffffu, mse[i], 2);
        sgn[i] += __shfl_xor_sync(0xffffffffu, sgn[i], 2);
      }
      logit_a[0] = nka * (mse[0] + gr.coef * rka * sgn[0]);
      logit_a[1] = nka * (mse[1] + gr.coef * rka * sgn[1]);
      logit_b[0] = nkb * (mse[2] + gr.coef * rkb * sgn[2]);
      logit_b[1] = nkb * (mse[3] + gr.coef * rkb * sgn[3]);
    }
    if constexpr (TWO) {
      const MmaGroup& gr = A.g[1];
      uint32_t ka[G1c::PK], kb_[G1c::PK];
      load_quarter<G1c::Q, G1c::PK>(gr.kcodes + sa * gr.kbytes, l, ka);
      load_quarter<G1c::Q, G1c::PK>(gr.kcodes + sb * gr.kbytes, l, kb_);
      load_quarter<G1c::Q, G1c::PV>(gr.vcodes + sa * gr.vbytes, l, vw1a);
      load_quarter<G1c::Q, G1c::PV>(gr.vcodes + sb * gr.vbytes, l, vw1b);
      const float nka = __half2float(__ushort_as_half(__ldg(gr.knorm + sa)));
      const float nkb = __half2float(__ushort_as_half(__ldg(gr.knorm + sb)));
      const float rka = __half2float(__ushort_as_half(__ldg(gr.krnorm + sa)));
      const float rkb = __half2float(__ushort_as_half(__ldg(gr.krnorm + sb)));
      nva1 = __half2float(__ushort_as_half(__ldg(gr.vnorm + sa)));
      nvb1 = __half2float(__ushort_as_half(__ldg(gr.vnorm + sb)));
      float mse[4], sgn[4];
      group_logits<G1c>(qf1, kl1, ka, kb_, mse, sgn);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mse[i] += __shfl_xor_sync(0xffffffffu, mse[i], 2);
        sgn[i] += __shfl_xor_sync(0xffffffffu, sgn[i], 2);
      }
      logit_a[0] += nka * (mse[0] + gr.coef * rka * sgn[0]);
      logit_a[1] += nka * (mse[1] + gr.coef * rka * sgn[1]);
      logit_b[0] += nkb * (mse[2] + gr.coef * rkb * sgn[2]);
      logit_b[1] += nkb * (mse[3] + gr.coef * rkb * sgn[3]);
    }
    // online softmax, log2 domain, heads h0 and h0+1 of this lane
    float la[2], lb[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      la[h] = va ? logit_a[h] * A.scale_log2 : -INFINITY;
      lb[h] = vb ? logit_b[h] * A.scale_log2 : -INFINITY;
    }
    float mt[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v = fmaxf(la[h], lb[h]);
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      mt[h] = v;
    }
    if (mt[0] > m_run[0] || mt[1] > m_run[1]) {
      float alpha[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float mn = fmaxf(m_run[h], mt[h]);
        alpha[h] = exp2f(m_run[h] - mn);
        m_run[h] = mn;
        l_run[h] *= alpha[h];
      }
#pragma unroll
      for (int i = 0; i < G0::NKB; ++i) {
        acc0[i][0] *= alpha[0]; acc0[i][1] *= alpha[1]; acc0[i][2] *= alpha[0]; acc0[i][3] *= alpha[1];
      }
      if constexpr (TWO) {
#pragma unroll
        for (int i = 0; i < G1c::NKB; ++i) {
          acc1[i][0] *= alpha[0]; acc1[i][1] *= alpha[1]; acc1[i][2] *= alpha[0]; acc1[i][3] *= alpha[1];
        }
      }
    }
    float pa[2], pb[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      pa[h] = exp2f(la[h] - m_run[h]);
      pb[h] = exp2f(lb[h] - m_run[h]);
      l_run[h] += pa[h] + pb[h];
    }
    // probability operand [P_hi | P_lo], weighted by each group's value norm
    auto pfrag = [&](float na, float nb, uint32_t& b0, uint32_t& b1) {
      float wa0 = pa[0] * na, wa1 = pa[1] * na, wb0 = pb[0] * nb, wb1 = pb[1] * nb;
      if (!hi_cols) {
        wa0 -= __half2float(__float2half_rn(wa0));
        wa1 -= __half2float(__float2half_rn(wa1));
        wb0 -= __half2float(__float2half_rn(wb0));
        wb1 -= __half2float(__float2half_rn(wb1));
      }
      b0 = movT(pack_h2(wa0, wa1));
      b1 = movT(pack_h2(wb0, wb1));
    };
    uint32_t pb0, pb1;
    pfrag(nva0, nvb0, pb0, pb1);
    group_values<G0>(vl0, vw0a, vw0b, pb0, pb1, acc0);
    if constexpr (TWO) {
      pfrag(nva1, nvb1, pb0, pb1);
      group_values<G1c>(vl1, vw1a, vw1b, pb0, pb1, acc1);
    }
  }

  // ---- warp state -> shared memory
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v = l_run[h];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    l_run[h] = v;
  }
  const int h0 = 2 * (l & 1);
  if (g == 0 && l < 2) {
    s_m[warp][h0] = m_run[0];
    s_m[warp][h0 + 1] = m_run[1];
    s_l[warp][h0] = l_run[0];
    s_l[warp][h0 + 1] = l_run[1];
  }
  auto store_acc = [&](auto& acc, auto gc_tag, int off) {
    using GC = decltype(gc_tag);
#pragma unroll
    for (int mb = 0; mb < GC::NKB; ++mb) {
      float v0 = acc[mb][0] + __shfl_xor_sync(0xffffffffu, acc[mb][0], 2);
      float v1 = acc[mb][1] + __shfl_xor_sync(0xffffffffu, acc[mb][1], 2);
      float v2 = acc[mb][2] + __shfl_xor_sync(0xffffffffu, acc[mb][2], 2);
      float v3 = acc[mb][3] + __shfl_xor_sync(0xffffffffu, acc[mb][3], 2);
      if (l < 2) {
        const int qq = mb & 3, hh = mb >> 2;
        const int c0 = GC::Q * (g >> 1) + qq + 16 * hh + 4 * (g & 1);   // row g: block f = 0
        const int c1 = c0 + 8;                                           // row g+8: block f = 1
        s_acc[warp][h0][off + c0] = v0;
        s_acc[warp][h0 + 1][off + c0] = v1;
        s_acc[warp][h0][off + c1] = v2;
        s_acc[warp][h0 + 1][off + c1] = v3;
      }
    }
  };
  store_acc(acc0, G0{}, A.g[0].off);
  if constexpr (TWO) store_acc(acc1, G1c{}, A.g[1].off);
  __syncthreads();
  // ---- merge the warps; one partial per (query head, split), m in natural-log units
  const float ln2 = 0.69314718055994531f;
  for (int e = threadIdx.x; e < kRep * A.D; e += blockDim.x) {
    const int h = e / A.D, c = e % A.D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][h]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = (s_m[w][h] == -INFINITY) ? 0.f : exp2f(s_m[w][h] - M);
      L += f * s_l[w][h];
      acc += f * s_acc[w][h][c];
    }
    float* dst = A.part + ((size_t)(b * A.Hq + hk * kRep + h) * A.nsplit + split) * (A.D + 2);
    if (c == 0) {
      dst[0] = (M == -INFINITY) ? -INFINITY : M * ln2;
      dst[1] = L;
    }
    dst[2 + c] = acc;
  }
}

template <class G0, class G1>
int launch_mma_t(const MmaArgs& A, int nsplit, int BHkv, cudaStream_t st) {
  dim3 grid(nsplit, BHkv);
  decode_mma_kernel<G0, G1><<<grid, kWarps * 32, 0, st>>>(A);
  count_launch();
  return check_launch("decode_mma_kernel");
}

}  // namespace

// Returns kNotHandled when the shape is outside this kernel's instantiations.
int launch_decode_mma(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G, const void* q,
                      int q_dtype, const tq_packed* kc, const tq_packed* vc, const int32_t* seq_lens, int B, int Hq,
                      int Hkv, int D, int64_t max_len, float scale, float* out, void* ws, cudaStream_t st) {
  if (Hq != kRep * Hkv || G > 2 || D > 256) return kNotHandled;
  int sig[2] = {0, 0};
  for (int g = 0; g < G; ++g) {
    const int dg = kctx[g]->lay.d;
    if (dg != 64 && dg != 128) return kNotHandled;
    if (vctx[g]->lay.k < 2) return kNotHandled;
    sig[g] = dg * 100 + kctx[g]->lay.k * 10 + vctx[g]->lay.k;
  }
  auto is = [&](int a, int bsig) { return sig[0] == a && sig[1] == bsig; };
  using C128_34 = GroupCfg<128, 3, 4>;
  using C64_34 = GroupCfg<64, 3, 4>;
  using C64_23 = GroupCfg<64, 2, 3>;
  using C64_12 = GroupCfg<64, 1, 2>;
  using C128_23 = GroupCfg<128, 2, 3>;
  const bool ok = (G == 1 && (sig[0] == 12834 || sig[0] == 12823)) || is(6434, 6423) || is(6423, 6412);
  if (!ok) return kNotHandled;

  int qp_ld = 0;
  for (int g = 0; g < G; ++g) qp_ld = std::max(qp_ld, kctx[g]->lay.d);
  int nsplit, chunk;
  decode_geometry(B, Hkv, max_len, &nsplit, &chunk);
  float* qprep = static_cast<float*>(ws);
  size_t qp_bytes = (size_t)B * Hq * G * 2 * qp_ld * sizeof(float);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + ((qp_bytes + 255) / 256) * 256);
  for (int g = 0; g < G; ++g) {
    int esz = q_dtype == TQ_DTYPE_F32 ? 4 : 2;
    const char* qg = static_cast<const char*>(q) + (size_t)off[g] * esz;
    int r = launch_prepare_queries(kctx[g], qg, q_dtype, (int64_t)B * Hq, D, qprep + (size_t)g * 2 * qp_ld,
                                   (int64_t)G * 2 * qp_ld, st);
    if (r != TQ_OK) return r;
  }
  MmaArgs A{};
  A.B = B; A.Hq = Hq; A.Hkv = Hkv; A.D = D; A.nsplit = nsplit; A.chunk = chunk; A.qp_ld = qp_ld; A.G = G;
  A.max_len = max_len; A.scale_log2 = scale * 1.4426950408889634f; A.seq_lens = seq_lens; A.qprep = qprep;
  A.part = part;
  for (int g = 0; g < G; ++g) {
    MmaGroup& gr = A.g[g];
    gr.kcodes = kc[g].codes; gr.knorm = kc[g].norm; gr.krnorm = kc[g].rnorm;
    gr.vcodes = vc[g].codes; gr.vnorm = vc[g].norm;
    for (int j = 0; j < 16; ++j) { gr.kc[j] = kctx[g]->cb.c[j]; gr.vc[j] = vctx[g]->cb.c[j]; }
    gr.coef = kctx[g]->sqrt_pi_over_2_over_m;
    gr.off = off[g];
    gr.kbytes = kctx[g]->lay.code_bytes;
    gr.vbytes = vctx[g]->lay.code_bytes;
  }
  int r;
  if (G == 1 && sig[0] == 12834) r = launch_mma_t<C128_34, void>(A, nsplit, B * Hkv, st);
  else if (G == 1) r = launch_mma_t<C128_23, void>(A, nsplit, B * Hkv, st);
  else if (is(6434, 6423)) r = launch_mma_t<C64_34, C64_23>(A, nsplit, B * Hkv, st);
  else r = launch_mma_t<C64_23, C64_12>(A, nsplit, B * Hkv, st);
  if (r != TQ_OK) return r;
  return launch_decode_merge(vctx, off, G, part, nsplit, B * Hq, D, out, st);
}

}  // namespace tq
