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
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

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

// Same, from a record staged in shared memory (byte offset of the record arbitrary: the
// staged copy keeps the global alignment of each record modulo 16).
template <int Q, int P>
__device__ __forceinline__ void lds_quarter(const uint8_t* rec, int l, uint32_t (&w)[P]) {
  if constexpr (Q == 32) {
    const uint8_t* p = rec + l * (4 * P);
    if constexpr (P == 4) {
      uint4 v = *reinterpret_cast<const uint4*>(p);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (P == 2) {
      uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    }
  } else {
    const uint8_t* p = rec + l * (2 * P);
    if constexpr (P == 4) {
      uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x & 0xFFFFu; w[1] = v.x >> 16; w[2] = v.y & 0xFFFFu; w[3] = v.y >> 16;
    } else if constexpr (P == 2) {
      uint32_t v = *reinterpret_cast<const uint32_t*>(p);
      w[0] = v & 0xFFFFu; w[1] = v >> 16;
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) w[i] = reinterpret_cast<const unsigned short*>(p)[i];
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

// fp16 centroid table split into low/high bytes, 8 entries per register pair (built on
// the host from the context's codebook).
struct Lut {
  uint32_t lo[4], hi[4];  // lo[0..1]: low bytes of c[0..7], lo[2..3]: of c[8..15]
};

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
  const float* PiV;    // value rotation [d_g][d_g] row-major (float32)
  Lut klut, vlut;      // fp16 key / value centroid tables
  float coef;          // sqrt(pi/2)/m
  int off;             // first channel of the group
  int kbytes, vbytes;  // record sizes
  int64_t kcap, vcap;  // slots allocated in the key / value caches
};

struct MmaArgs {
  MmaGroup g[2];
  int B, Hq, Hkv, D, nsplit, chunk, qp_ld, G;
  int64_t max_len;
  float scale_log2;    // softmax scale * log2(e)
  const int32_t* seq_lens;
  const float* qprep;  // [B*Hq][G][2*qp_ld]: (Pi q, S q) of each group
  float* part;         // [B*Hq][nsplit][D+2]: (m, l, acc) per split
  float* out;          // [B*Hq][D]
  int* err;            // device error word (a pipeline wait that timed out)
};

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void allow_dependent_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Query fragments of one group for this thread, built once per CTA.
template <class GC>
struct QFrag {
  uint32_t mse[GC::NKB][2];
  uint32_t sgn[GC::NKB][2];
};

template <class GC>
__device__ __forceinline__ void load_qfrag(QFrag<GC>& f, const MmaArgs& A, int gi, int b, int hk, int lane) {
  const int g = lane >> 2, l = lane & 3;
  const int head = hk * kRep + (g >> 1);   // column n = g: head n/2, hi (n even) or lo (n odd) half
  const bool lo_part = (g & 1) != 0;
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
      // rows (coordinates) g: block f = 0, g+8: block f = 1; k (tokens) 2l.. from token g, 2l+8.. from g+8
      mma16816(acc[mb], movT(x0f), movT(x0s), movT(x1f), movT(x1s), pb0, pb1);
    }
  }
}

// Everything a thread loads for one 16-token tile of one group.
template <class GC>
struct TileData {
  uint32_t ka[GC::PK], kb[GC::PK], va[GC::PV], vb[GC::PV];
  unsigned short nka, nkb, rka, rkb, nva, nvb;
};

template <class GC>
__device__ __forceinline__ void load_tile(TileData<GC>& t, const MmaGroup& gr, int64_t sa, int64_t sb, int l) {
  load_quarter<GC::Q, GC::PK>(gr.kcodes + sa * gr.kbytes, l, t.ka);
  load_quarter<GC::Q, GC::PK>(gr.kcodes + sb * gr.kbytes, l, t.kb);
  load_quarter<GC::Q, GC::PV>(gr.vcodes + sa * gr.vbytes, l, t.va);
  load_quarter<GC::Q, GC::PV>(gr.vcodes + sb * gr.vbytes, l, t.vb);
  t.nka = __ldg(gr.knorm + sa);
  t.nkb = __ldg(gr.knorm + sb);
  t.rka = __ldg(gr.krnorm + sa);
  t.rkb = __ldg(gr.krnorm + sb);
  t.nva = __ldg(gr.vnorm + sa);
  t.nvb = __ldg(gr.vnorm + sb);
}

__device__ __forceinline__ float h2f(unsigned short h) { return __half2float(__ushort_as_half(h)); }

template <class GC>
__device__ __forceinline__ void tile_logits(const TileData<GC>& t, const QFrag<GC>& qf, const Lut& kl,
                                            const MmaGroup& gr, float& la, float& lb) {
  float mse[4], sgn[4];
  group_logits<GC>(qf, kl, t.ka, t.kb, mse, sgn);
  // columns 2l, 2l+1 are the hi and lo halves of head l
  const float ca = gr.coef * h2f(t.rka), cb = gr.coef * h2f(t.rkb);
  la += h2f(t.nka) * fmaf(ca, sgn[0] + sgn[1], mse[0] + mse[1]);
  lb += h2f(t.nkb) * fmaf(cb, sgn[2] + sgn[3], mse[2] + mse[3]);
}

constexpr int kStageTok = kWarps * 16;  // tokens per pipeline stage: one 16-token tile per consumer warp
constexpr int kNStage = 4;
constexpr uint64_t kDecWaitNs = 2000000000ull;

// Shared-memory layout of one pipeline stage: per group the K and V code bytes of 64
// consecutive slots (copied with 16-byte granularity, hence 32 bytes of slack) and the
// three fp16 norm arrays.
template <class G0, class G1c, bool TWO>
struct Stage {
  static constexpr int KB0 = G0::PK * G0::DG / 8, VB0 = G0::PV * G0::DG / 8;
  static constexpr int KB1 = G1c::PK * G1c::DG / 8, VB1 = G1c::PV * G1c::DG / 8;
  static constexpr int OFF_K0 = 0;
  static constexpr int OFF_V0 = OFF_K0 + kStageTok * KB0 + 32;
  static constexpr int OFF_K1 = OFF_V0 + kStageTok * VB0 + 32;
  static constexpr int OFF_V1 = OFF_K1 + (TWO ? kStageTok * KB1 + 32 : 0);
  static constexpr int OFF_N = OFF_V1 + (TWO ? kStageTok * VB1 + 32 : 0);   // uint16 [G][3][64]
  static constexpr int BYTES = ((OFF_N + (TWO ? 2 : 1) * 3 * kStageTok * 2) + 127) / 128 * 128;
};

// Copy bytes [b0, b1) of a packed array into shared memory at dst + (b0 & 15): one bulk copy
// of the 16-byte aligned span inside the allocation, plain loads for a ragged end beyond
// the last full 16 bytes of the allocation.  Returns the bulk byte count (for expect_tx).
__device__ __forceinline__ uint32_t stage_span(uint8_t* dst, const uint8_t* src, int64_t b0, int64_t b1, int64_t total,
                                               uint64_t* bar, bool issue) {
  const int64_t a0 = b0 & ~int64_t(15);
  const int64_t cap16 = total & ~int64_t(15);
  int64_t a1 = (b1 + 15) & ~int64_t(15);
  if (a1 > cap16) a1 = cap16;
  uint32_t bytes = a1 > a0 ? (uint32_t)(a1 - a0) : 0u;
  if (issue) {
    if (bytes) bulk_load(dst, src + a0, bytes, bar);
    for (int64_t x = (a1 > a0 ? a1 : a0); x < b1; ++x) dst[x - a0] = src[x];
  }
  return bytes;
}

template <class G0, class G1>
__global__ void __launch_bounds__((kWarps + 1) * 32, 3) decode_mma_kernel(MmaArgs A) {
  constexpr bool TWO = !std::is_same<G1, void>::value;
  using G1c = typename std::conditional<TWO, G1, G0>::type;
  using ST = Stage<G0, G1c, TWO>;
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ float s_m[kWarps][kRep], s_l[kWarps][kRep];
  __shared__ float s_acc[kWarps][kRep][256];
  __shared__ __align__(8) uint64_t full[kNStage], empty[kNStage];
  __shared__ int s_abort;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / A.Hkv, hk = bh % A.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int T = max(0, (int)min((int64_t)A.seq_lens[b], A.max_len));
  const int t_begin = split * A.chunk;
  const int t_end = min(T, t_begin + A.chunk);
  const int64_t slot0 = (int64_t)bh * A.max_len;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNStage; ++i) {
      mbar_init(full + i, 32);
      mbar_init(empty + i, kWarps);
    }
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const volatile int* abort_v = &s_abort;
  auto fail = [&](int code) {
    atomicExch(&s_abort, 1);
    if (A.err) atomicCAS(A.err, 0, code);
  };

  if (warp == kWarps) {
    // ---------------------------------------------------------------- producer warp
    int it = 0;
    int pending[kNStage];
    for (int i = 0; i < kNStage; ++i) pending[i] = -1;
    for (int ts = t_begin; ts < t_end; ts += kStageTok, ++it) {
      const int s = it % kNStage;
      const uint32_t ph = (it / kNStage) & 1;
      if (!mbar_wait(empty + s, ph ^ 1, abort_v, kDecWaitNs)) { fail(201); break; }
      const int ntok = min(kStageTok, t_end - ts);
      uint8_t* st = dsm + s * ST::BYTES;
      const int64_t first = slot0 + ts, last = slot0 + ts + ntok;
      auto spans = [&](bool issue) {
        uint32_t tx = 0;
        const MmaGroup& g0 = A.g[0];
        tx += stage_span(st + ST::OFF_K0, g0.kcodes, first * ST::KB0, last * ST::KB0, g0.kcap * ST::KB0, full + s, issue);
        tx += stage_span(st + ST::OFF_V0, g0.vcodes, first * ST::VB0, last * ST::VB0, g0.vcap * ST::VB0, full + s, issue);
        if constexpr (TWO) {
          const MmaGroup& g1 = A.g[1];
          tx += stage_span(st + ST::OFF_K1, g1.kcodes, first * ST::KB1, last * ST::KB1, g1.kcap * ST::KB1, full + s, issue);
          tx += stage_span(st + ST::OFF_V1, g1.vcodes, first * ST::VB1, last * ST::VB1, g1.vcap * ST::VB1, full + s, issue);
        }
        return tx;
      };
      if (lane == 0) {
        mbar_expect_tx(full + s, spans(false));
        spans(true);
      }
      uint16_t* nrm = reinterpret_cast<uint16_t*>(st + ST::OFF_N);
      for (int j = lane; j < kStageTok; j += 32) {
        const bool ok = j < ntok;
        const int64_t sl = slot0 + ts + j;
#pragma unroll
        for (int gi = 0; gi < (TWO ? 2 : 1); ++gi) {
          const MmaGroup& gr = A.g[gi];
          nrm[(gi * 3 + 0) * kStageTok + j] = ok ? __ldg(gr.knorm + sl) : (uint16_t)0;
          nrm[(gi * 3 + 1) * kStageTok + j] = ok ? __ldg(gr.krnorm + sl) : (uint16_t)0;
          nrm[(gi * 3 + 2) * kStageTok + j] = ok ? __ldg(gr.vnorm + sl) : (uint16_t)0;
        }
      }
      __syncwarp();
      mbar_arrive(full + s);
      if (lane == 0) pending[s] = (int)ph;
    }
    // bulk copies still in flight land before the CTA exits
    if (lane == 0)
      for (int i = 0; i < kNStage; ++i)
        if (pending[i] >= 0) mbar_wait(full + i, (uint32_t)pending[i], nullptr, kDecWaitNs);
  }

  // ------------------------------------------------------------------ consumer warps
  float acc0[G0::NKB][4];
  float acc1[G1c::NKB][4];
  float m_run = -INFINITY, l_run = 0.f;
  if (warp < kWarps) {
    const Lut kl0 = A.g[0].klut, vl0 = A.g[0].vlut;
    const Lut kl1 = A.g[TWO ? 1 : 0].klut, vl1 = A.g[TWO ? 1 : 0].vlut;
    grid_dependency_wait();   // prepared queries come from the preceding kernel
    QFrag<G0> qf0;
    load_qfrag<G0>(qf0, A, 0, b, hk, lane);
    QFrag<G1c> qf1;
    if constexpr (TWO) load_qfrag<G1c>(qf1, A, 1, b, hk, lane);
#pragma unroll
    for (int i = 0; i < G0::NKB; ++i) acc0[i][0] = acc0[i][1] = acc0[i][2] = acc0[i][3] = 0.f;
#pragma unroll
    for (int i = 0; i < G1c::NKB; ++i) acc1[i][0] = acc1[i][1] = acc1[i][2] = acc1[i][3] = 0.f;
    int it = 0;
    for (int ts = t_begin; ts < t_end; ts += kStageTok, ++it) {
      const int s = it % kNStage;
      if (!mbar_wait(full + s, (it / kNStage) & 1, abort_v, kDecWaitNs)) { fail(202); break; }
      const int tt = ts + warp * 16;           // this warp's 16-token tile
      const bool live = tt < t_end;
      const uint8_t* st = dsm + s * ST::BYTES;
      const int64_t first = slot0 + ts;
      const int ja = warp * 16 + g, jb = ja + 8;   // stage-local token rows of this lane
      TileData<G0> c0;
      TileData<G1c> c1;
      if (live) {
        const uint8_t* k0 = st + ST::OFF_K0 + ((first * ST::KB0) & 15);
        const uint8_t* v0 = st + ST::OFF_V0 + ((first * ST::VB0) & 15);
        lds_quarter<G0::Q, G0::PK>(k0 + ja * ST::KB0, l, c0.ka);
        lds_quarter<G0::Q, G0::PK>(k0 + jb * ST::KB0, l, c0.kb);
        lds_quarter<G0::Q, G0::PV>(v0 + ja * ST::VB0, l, c0.va);
        lds_quarter<G0::Q, G0::PV>(v0 + jb * ST::VB0, l, c0.vb);
        const uint16_t* nrm = reinterpret_cast<const uint16_t*>(st + ST::OFF_N);
        c0.nka = nrm[ja]; c0.nkb = nrm[jb];
        c0.rka = nrm[kStageTok + ja]; c0.rkb = nrm[kStageTok + jb];
        c0.nva = nrm[2 * kStageTok + ja]; c0.nvb = nrm[2 * kStageTok + jb];
        if constexpr (TWO) {
          const uint8_t* k1 = st + ST::OFF_K1 + ((first * ST::KB1) & 15);
          const uint8_t* v1 = st + ST::OFF_V1 + ((first * ST::VB1) & 15);
          lds_quarter<G1c::Q, G1c::PK>(k1 + ja * ST::KB1, l, c1.ka);
          lds_quarter<G1c::Q, G1c::PK>(k1 + jb * ST::KB1, l, c1.kb);
          lds_quarter<G1c::Q, G1c::PV>(v1 + ja * ST::VB1, l, c1.va);
          lds_quarter<G1c::Q, G1c::PV>(v1 + jb * ST::VB1, l, c1.vb);
          c1.nka = nrm[3 * kStageTok + ja]; c1.nkb = nrm[3 * kStageTok + jb];
          c1.rka = nrm[4 * kStageTok + ja]; c1.rkb = nrm[4 * kStageTok + jb];
          c1.nva = nrm[5 * kStageTok + ja]; c1.nvb = nrm[5 * kStageTok + jb];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);   // the stage's data now sits in registers
      if (!live) continue;
      float la = 0.f, lb = 0.f;
      tile_logits<G0>(c0, qf0, kl0, A.g[0], la, lb);
      if constexpr (TWO) tile_logits<G1c>(c1, qf1, kl1, A.g[1], la, lb);
      // online softmax (log2 domain) of head l over tokens g, g+8 of the tile
      la = (tt + g < t_end) ? la * A.scale_log2 : -INFINITY;
      lb = (tt + g + 8 < t_end) ? lb * A.scale_log2 : -INFINITY;
      float mt = fmaxf(la, lb);
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      if (mt > m_run) {
        const float alpha = exp2f(m_run - mt);
        m_run = mt;
        l_run *= alpha;
#pragma unroll
        for (int i = 0; i < G0::NKB; ++i) {
          acc0[i][0] *= alpha; acc0[i][1] *= alpha; acc0[i][2] *= alpha; acc0[i][3] *= alpha;
        }
        if constexpr (TWO) {
#pragma unroll
          for (int i = 0; i < G1c::NKB; ++i) {
            acc1[i][0] *= alpha; acc1[i][1] *= alpha; acc1[i][2] *= alpha; acc1[i][3] *= alpha;
          }
        }
      }
      const float pa = exp2f(la - m_run), pb = exp2f(lb - m_run);
      l_run += pa + pb;
      auto pfrag = [&](float na, float nb, uint32_t& b0, uint32_t& b1) {
        const float wa = pa * na, wb = pb * nb;
        const float ha = __half2float(__float2half_rn(wa)), hb = __half2float(__float2half_rn(wb));
        b0 = movT(pack_h2(ha, wa - ha));
        b1 = movT(pack_h2(hb, wb - hb));
      };
      uint32_t pb0, pb1;
      pfrag(h2f(c0.nva), h2f(c0.nvb), pb0, pb1);
      group_values<G0>(vl0, c0.va, c0.vb, pb0, pb1, acc0);
      if constexpr (TWO) {
        pfrag(h2f(c1.nva), h2f(c1.nvb), pb0, pb1);
        group_values<G1c>(vl1, c1.va, c1.vb, pb0, pb1, acc1);
      }
    }
    // ---- warp state -> shared memory (lane (g, l) holds head l)
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
    if (g == 0) {
      s_m[warp][l] = m_run;
      s_l[warp][l] = l_run;
    }
    auto store_acc = [&](auto& acc, auto gc_tag, int off) {
      using GC = decltype(gc_tag);
#pragma unroll
      for (int mb = 0; mb < GC::NKB; ++mb) {
        const int qq = mb & 3, hh = mb >> 2;
        const int c0_ = GC::Q * (g >> 1) + qq + 16 * hh + 4 * (g & 1);   // row g: block f = 0
        s_acc[warp][l][off + c0_] = acc[mb][0] + acc[mb][1];
        s_acc[warp][l][off + c0_ + 8] = acc[mb][2] + acc[mb][3];          // row g+8: block f = 1
      }
    };
    store_acc(acc0, G0{}, A.g[0].off);
    if constexpr (TWO) store_acc(acc1, G1c{}, A.g[1].off);
  }
  __syncthreads();
  // ---- merge the warps: one partial per (query head, split); m in natural-log units
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
  // the merge kernel (launched programmatically behind this one) may start once every
  // CTA has written its partial
  __syncthreads();
  allow_dependent_launch();
}

// (Pi q, S q) of the kRep query heads of one (sequence, kv head), 64 outputs per CTA
// (blockIdx.y selects them; outputs o < d_g are Pi q, the rest S q): the 64 needed
// columns of Pi^T or S^T are staged in shared memory with 16-byte loads, then thread
// (head, o) takes its dot product from shared memory.
template <typename T>
__global__ void __launch_bounds__(256) decode_prep_kernel(const T* __restrict__ q, int D, int off, int dg,
                                                          const float* __restrict__ PiT, const float* __restrict__ ST,
                                                          float* __restrict__ qprep, int G, int gi, int qp_ld) {
  __shared__ __align__(16) float ms[128 * 64];
  __shared__ float qs[kRep][128];
  allow_dependent_launch();
  const int grp = blockIdx.x;                    // = b * Hkv + hk; rows grp*kRep .. +kRep-1
  const int o0 = blockIdx.y * 64;                // first output of this CTA
  const float* M = o0 < dg ? PiT + o0 : ST + (o0 - dg);
  float4* m4 = reinterpret_cast<float4*>(ms);
#pragma unroll 8
  for (int e = threadIdx.x; e < dg * 16; e += blockDim.x) {     // dg rows x 16 float4
    const int j = e >> 4, c4 = e & 15;
    m4[e] = __ldg(reinterpret_cast<const float4*>(M + (size_t)j * dg) + c4);
  }
  for (int e = threadIdx.x; e < kRep * dg; e += blockDim.x) {
    const int h = e / dg, j = e % dg;
    const size_t at = (size_t)(grp * kRep + h) * D + off + j;
    if constexpr (std::is_same<T, float>::value) qs[h][j] = q[at];
    else qs[h][j] = __bfloat162float(q[at]);
  }
  __syncthreads();
  const int h = threadIdx.x >> 6, oc = threadIdx.x & 63;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
  for (int j = 0; j < dg; j += 2) {
    a0 = fmaf(ms[j * 64 + oc], qs[h][j], a0);
    a1 = fmaf(ms[(j + 1) * 64 + oc], qs[h][j + 1], a1);
  }
  qprep[((size_t)(grp * kRep + h) * G + gi) * 2 * qp_ld + o0 + oc] = a0 + a1;
}

// Log-sum-exp merge of the context splits and the inverse rotation of the value groups:
// one CTA per (query row, 64 output channels).  The merged rotated-basis accumulator of
// the row is built in shared memory (all splits' loads independent), then thread
// (output, quarter) sums a quarter of o[c] = sum_i Pi_v[i][c - off] acc[off + i].
struct Merge2Args {
  const float* part;
  int nsplit, D, G;
  int off[3];
  const float* PiV[2];
  float* out;
};

__global__ void __launch_bounds__(256) decode_merge_mma_kernel(Merge2Args A) {
  __shared__ float w[512];
  __shared__ float acc[256];
  __shared__ float red[4][64];
  __shared__ float part2[2][256];
  grid_dependency_wait();
  const int row = blockIdx.x, c0 = blockIdx.y * 64;
  const int D = A.D, ns = A.nsplit;
  const float* P = A.part + (size_t)row * ns * (D + 2);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, P[(size_t)s * (D + 2)]);
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = P[(size_t)s * (D + 2)];
      const float f = (ms == -INFINITY) ? 0.f : __expf(ms - M);
      w[s] = f;
      L += f * P[(size_t)s * (D + 2) + 1];
    }
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __syncwarp();
    for (int s = lane; s < ns; s += 32) w[s] *= inv;
  }
  __syncthreads();
  // every split's contribution is an independent load: keep 16 of them in flight per thread
  {
    const int nthr = blockDim.x;
    const int halves = nthr / D > 1 ? nthr / D : 1;     // threads per coordinate
    const int i = threadIdx.x % D, hsel = threadIdx.x / D;
    float a[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) a[u] = 0.f;
    if (hsel < halves) {
      for (int s0 = hsel * 16; s0 < ns; s0 += 16 * halves) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (s0 + u < ns) a[u] = fmaf(w[s0 + u], P[(size_t)(s0 + u) * (D + 2) + 2 + i], a[u]);
      }
    }
    float t = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) t += a[u];
    if (hsel < halves) part2[hsel][i] = t;
    __syncthreads();
    if (hsel == 0) {
      float sum = 0.f;
      for (int h = 0; h < halves; ++h) sum += part2[h][i];
      acc[i] = sum;
    }
  }
  __syncthreads();
  const int oc = threadIdx.x & 63, qtr = threadIdx.x >> 6;
  const int c = c0 + oc;
  float o = 0.f;
  if (c < D) {
    const int gi = (A.G > 1 && c >= A.off[1]) ? 1 : 0;
    const int off = A.off[gi], dg = A.off[gi + 1] - off, j = c - off;
    const float* Pi = A.PiV[gi] + j;
    const int i0 = qtr * (dg / 4), i1 = i0 + dg / 4;
#pragma unroll 8
    for (int i = i0; i < i1; ++i) o = fmaf(__ldg(Pi + (size_t)i * dg), acc[off + i], o);
  }
  red[qtr][oc] = o;
  __syncthreads();
  if (qtr == 0 && c < D)
    A.out[(size_t)row * D + c] = (red[0][oc] + red[1][oc]) + (red[2][oc] + red[3][oc]);
}

template <class G0, class G1>
int launch_mma_t(const MmaArgs& A, int nsplit, int BHkv, cudaStream_t st) {
  constexpr bool TWO = !std::is_same<G1, void>::value;
  using G1c = typename std::conditional<TWO, G1, G0>::type;
  const int dyn = kNStage * Stage<G0, G1c, TWO>::BYTES;
  cudaError_t ea = cudaFuncSetAttribute(decode_mma_kernel<G0, G1>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (ea != cudaSuccess) return cuda_fail(ea, "cudaFuncSetAttribute(decode_mma_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsplit, BHkv);
  cfg.blockDim = dim3((kWarps + 1) * 32);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_mma_kernel<G0, G1>, A);
  count_launch();
  if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(decode_mma_kernel)");
  return check_launch("decode_mma_kernel");
}

}  // namespace

Lut host_lut(const Codebook& cb) {
  Lut t{};
  for (int j = 0; j < 16; ++j) {
    uint16_t b = 0;
    if (j < cb.K) {
      __half h = __float2half_rn(cb.c[j]);
      b = *reinterpret_cast<uint16_t*>(&h);
    }
    t.lo[j / 4] |= (uint32_t)(b & 0xFF) << (8 * (j % 4));
    t.hi[j / 4] |= (uint32_t)(b >> 8) << (8 * (j % 4));
  }
  return t;
}

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

  const DecodeWs W = decode_ws(B, Hq, Hkv, D, G, max_len);
  if (W.nsplit > 512) return kNotHandled;
  char* base = static_cast<char*>(ws);
  float* qprep = reinterpret_cast<float*>(base + W.qp);
  float* part = reinterpret_cast<float*>(base + W.part);
  for (int g = 0; g < G; ++g) {
    const int dg = kctx[g]->lay.d;
    const dim3 pgrid(B * Hkv, 2 * dg / 64);
    if (q_dtype == TQ_DTYPE_F32)
      decode_prep_kernel<float><<<pgrid, 256, 0, st>>>(static_cast<const float*>(q), D, off[g], dg, kctx[g]->PiT,
                                                       kctx[g]->ST, qprep, G, g, D);
    else
      decode_prep_kernel<__nv_bfloat16><<<pgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), D, off[g], dg,
                                                               kctx[g]->PiT, kctx[g]->ST, qprep, G, g, D);
    count_launch();
    int r = check_launch("decode_prep_kernel");
    if (r != TQ_OK) return r;
  }
  MmaArgs A{};
  A.B = B; A.Hq = Hq; A.Hkv = Hkv; A.D = D; A.nsplit = W.nsplit; A.chunk = W.chunk; A.qp_ld = D; A.G = G;
  A.max_len = max_len; A.scale_log2 = scale * 1.4426950408889634f; A.seq_lens = seq_lens; A.qprep = qprep;
  A.part = part; A.out = out;
  for (int g = 0; g < G; ++g) {
    MmaGroup& gr = A.g[g];
    gr.kcodes = kc[g].codes; gr.knorm = kc[g].norm; gr.krnorm = kc[g].rnorm;
    gr.vcodes = vc[g].codes; gr.vnorm = vc[g].norm;
    gr.PiV = vctx[g]->Pi;
    gr.klut = host_lut(kctx[g]->cb);
    gr.vlut = host_lut(vctx[g]->cb);
    gr.coef = kctx[g]->sqrt_pi_over_2_over_m;
    gr.off = off[g];
    gr.kbytes = kctx[g]->lay.code_bytes;
    gr.vbytes = vctx[g]->lay.code_bytes;
    gr.kcap = kc[g].cap;
    gr.vcap = vc[g].cap;
  }
  A.err = kctx[0]->dev_err;
  int r;
  if (G == 1 && sig[0] == 12834) r = launch_mma_t<C128_34, void>(A, W.nsplit, B * Hkv, st);
  else if (G == 1) r = launch_mma_t<C128_23, void>(A, W.nsplit, B * Hkv, st);
  else if (is(6434, 6423)) r = launch_mma_t<C64_34, C64_23>(A, W.nsplit, B * Hkv, st);
  else r = launch_mma_t<C64_23, C64_12>(A, W.nsplit, B * Hkv, st);
  if (r != TQ_OK) return r;
  Merge2Args M{};
  M.part = part; M.nsplit = W.nsplit; M.D = D; M.G = G; M.out = out;
  for (int g = 0; g < G; ++g) { M.off[g] = off[g]; M.PiV[g] = vctx[g]->Pi; }
  M.off[G] = D;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * Hq, div_up(D, 64));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_merge_mma_kernel, M);
  count_launch();
  if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(decode_merge_mma_kernel)");
  return check_launch("decode_merge_mma_kernel");
}

}  // namespace tq
