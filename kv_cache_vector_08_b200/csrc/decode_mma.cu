// Decode attention over the packed cache on the tensor cores, operands built in registers.
//
// turboquant.net "集成到 Attention": keys and values stay quantized and attention reads
// them directly; admirer.cn (H100 paragraph): the attention-logit computation on 4-bit
// keys is where the speed-up is measured.  Per cached token and GQA group of query heads
// the work is a small contraction (4 heads x d coordinates for the MSE term, the QJL sign
// term and the value accumulation), so each warp runs it on mma.sync over 16-token tiles:
//
//   keys (int8, m16n8k32):  [16 tokens x 32 coords] x [32 coords x 8]
//      MSE term  C_hi * Q~ + C_lo * Q~    centroids as two int8 digits of a 16-bit fixed
//                                          point, the prepared query Pi q as two int8
//                                          digits in the 8 columns (4 heads x hi/lo)
//      QJL term  A_s * Q^                 A_s = -[sign bit], from one sign-replicating
//                                          byte permute per 4 coordinates
//   values (fp16, m16n8k16): out^T [16 coords x 8] += Cv^T [16 x 16 tokens] * [P_hi | P_lo]
//
// The A operands come straight from the packed words: for every 8-coordinate slice the
// low code bits are nibbles of one word (one AND gives four byte-permute selectors) and
// the top bits sit at byte msbs after at most one shift, so a 4-entry byte lookup costs
// one prmt.  Keys: the two centroid digits are two lookups, the sign bytes one prmt.
// Values: magnitude bytes are looked up (low and high byte of the fp16 magnitude), the
// negative flag is XORed into the sign bit, two prmt interleave the bytes, movmatrix turns
// the 8x8 blocks around.  Integer products are exact; the fixed-point scales (max |v| of
// each prepared query row, max |c| for the centroids) keep every digit in range, so the
// logits carry only the 2^-15 rounding of the two fixed-point operands.
//
// Three kernels, linked by programmatic dependent launch: the prep kernel rotates the
// queries (fp32, one warp per 8 rows x 8 outputs, small enough to share an SM with the
// decode CTAs, which start at once and stream their first stages meanwhile); the decode
// kernel, where one CTA (4 consumer warps + 1 producer warp) handles one (sequence, kv
// head, context split): the producer stages 64 tokens of K/V code bytes and norms per
// pipeline stage with bulk copies, consumer warps form the query digits, take one 16-token
// tile of every stage, keep an online softmax (log2 domain) per head, and merge their
// states in shared memory before writing one partial (m, l, acc) per query head and split;
// and the merge kernel (log-sum-exp over the splits, then the inverse value rotation).
#include <algorithm>
#include <cfloat>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_ops.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;
using namespace mmaops;

constexpr int kWarps = 4;
constexpr int kRep = 4;            // query heads per kv head handled by this kernel
#ifndef TQ_DECODE_CTAS_PER_SM
#define TQ_DECODE_CTAS_PER_SM 3    // resident decode CTAs per SM the register budget is sized for
#endif

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
template <int DG_, int PK_, int PV_>
struct GroupCfg {
  static constexpr int DG = DG_;            // group width (64 or 128)
  static constexpr int PK = PK_;            // key code bits (MSE index bits + QJL sign)
  static constexpr int PV = PV_;            // value code bits
  static constexpr int NS = DG_ / 32;       // 8-coordinate slices per thread
  static constexpr int CQ = DG_ / 4;        // coordinates per thread
  static constexpr int KB = PK_ * DG_ / 8;  // key record bytes
  static constexpr int VB = PV_ * DG_ / 8;  // value record bytes
};

// The words of one record a thread needs: d = 128, its own 32-coordinate block (P words);
// d = 64 with P = 4, its two slices' words; d = 64 otherwise, the block it shares with its
// neighbour (P words), pre-shifted so that slice u of this thread reads like slice u of a
// d = 128 block (the shared words interleave the two threads' slices).
template <int DG, int P>
struct Words {
  static constexpr int N = (DG == 64 && P == 4) ? 2 : P;
  uint32_t w[N];
};

template <int DG, int P>
__device__ __forceinline__ void lds_words(Words<DG, P>& r, const uint8_t* rec, int l) {
  if constexpr (DG == 128 && P == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(rec + 16 * l);
    r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
  } else if constexpr (DG == 64 && P == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(rec + 8 * l);
    r.w[0] = v.x; r.w[1] = v.y;
  } else if constexpr (DG == 128) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(rec + 4 * P * l);
#pragma unroll
    for (int i = 0; i < P; ++i) r.w[i] = p[i];
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(rec + 4 * P * (l >> 1));
#pragma unroll
    for (int i = 0; i < P; ++i) r.w[i] = p[i];
    const int odd = l & 1;                    // this thread's slices are 2*odd, 2*odd+1
    if constexpr (P == 3) {
      r.w[0] >>= 2 * odd;
      r.w[1] >>= 2 * odd;
    } else {
      r.w[0] >>= 2 * odd;
    }
    r.w[P - 1] <<= 4 * odd;
  }
}

// Byte-permute selectors (low code bits) of slice u: nibbles 0-3 = coordinates 8u..8u+3,
// nibbles 4-7 = 8u+4..8u+7 of this thread.
template <int DG, int P>
__device__ __forceinline__ uint32_t low_sel(const Words<DG, P>& r, int u) {
  if constexpr (P == 4) return r.w[u] & 0x77777777u;
  else if constexpr (P == 3) return (r.w[u & 1] >> (2 * (u >> 1))) & 0x33333333u;
  else return (r.w[0] >> u) & 0x11111111u;
}

// Top code bits of slice u, half h (coordinates 8u + 4h + t) at the msbs of bytes t.
template <int DG, int P>
__device__ __forceinline__ uint32_t top_bits(const Words<DG, P>& r, int u, int h) {
  if constexpr (P == 4) return h ? (r.w[u] << 4) : r.w[u];
  else return r.w[P - 1] << (2 * u + h);
}

// Per-group kernel arguments.
struct MmaGroup {
  const uint8_t* kcodes;
  const uint16_t* knorm;
  const uint16_t* krnorm;
  const uint8_t* vcodes;
  const uint16_t* vnorm;
  Luts lut;
  float kc_inv;        // 1 / key-centroid fixed-point scale
  float coef;          // sqrt(pi/2)/m
  int off;             // first channel of the group
  int64_t kcap, vcap;  // slots allocated in the key / value caches
};

struct MmaArgs {
  MmaGroup g[2];
  int B, Hq, Hkv, D, nsplit, chunk, G;
  int rep, nsub;           // query heads per kv head; CTAs per (sequence, kv head) = ceil(rep / 4)
  int64_t max_len;
  float scale_log2;        // softmax scale * log2(e)
  const int32_t* seq_lens;
  const float* qprep;      // [B*Hq][G][2][D]: Pi q, S q of every group (fp32)
  float* part;             // [B*Hq] rows of part_ld floats: [nsplit][D+2] (m, l, acc) per split
  int64_t part_ld;
  int* err;                // device error word (a pipeline wait that timed out)
  const float* piv[2];     // value-group rotations, read by the merge kernel: prefetched
  uint32_t piv_bytes[2];   // into L2 at the start of this kernel
  const int32_t* table;    // paged cache: physical page of (sequence, logical page), or NULL
  int page, max_pages;     // tokens per page (a multiple of the 64-token stage), pages per sequence
  int64_t npages;          // physical pages the caches hold (min over the groups' caches)
};

// First cache slot of the 64-token stage starting at token ts of (sequence b, kv head hk).
// Contiguous caches: slot0 + ts.  Paged caches: page p of the pool holds kv head hk's
// tokens in slots (p Hkv + hk) page .. + page - 1; a stage never crosses a page.  A page
// index outside the pool reads page 0 and is reported as device error 901.
__device__ __forceinline__ int64_t stage_slot(const MmaArgs& A, int b, int hk, int ts, int64_t slot0) {
  if (!A.table) return slot0 + ts;
  int pg = __ldg(A.table + (size_t)b * A.max_pages + ts / A.page);
  if (pg < 0 || pg >= A.npages) {
    if (A.err) atomicCAS(A.err, 0, (int)kErrSlotRange);
    pg = 0;
  }
  return ((int64_t)pg * A.Hkv + hk) * A.page + ts % A.page;
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Query head of MMA column group j (0..3) of a CTA that serves heads sub*4 .. sub*4+3 of kv
// head hk; columns past the kv head's rep heads repeat its last head (their results are
// not written).
__device__ __forceinline__ int col_head(int hk, int rep, int sub, int j) {
  return hk * rep + min(sub * kRep + j, rep - 1);
}
__device__ __forceinline__ void allow_dependent_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Query operands of one group for this thread: B fragments (column g = head g/2, digit
// g&1; k-slots = this thread's coordinates 8u + 4h + t), and, for the thread's own
// accumulator head l, the fixed-point scales and sum_j Q^_j (for the QJL identity).
template <class GC>
struct QOps {
  uint32_t bm[GC::NS][2], bs[GC::NS][2];
  float inv_m, inv_s, sum_s;
};

template <class GC>
__device__ __forceinline__ void load_qops(QOps<GC>& f, const MmaArgs& A, int gi, int b, int hk, int sub, int lane) {
  const int g = lane >> 2, l = lane & 3;
  const int head = col_head(hk, A.rep, sub, g >> 1);
  const bool lo = (g & 1) != 0;
  const float* pm = A.qprep + ((size_t)(b * A.Hq + head) * A.G + gi) * 2 * A.D + GC::CQ * l;
  const float* ps = pm + A.D;
  // fixed-point scale of each (head, part) row: 32000 / max |v| over the group's
  // coordinates (the four threads of a quad hold the head's d_g coordinates); all of the
  // thread's values are loaded in one round
  float4 va[GC::CQ / 4], vc[GC::CQ / 4];
#pragma unroll
  for (int u = 0; u < GC::CQ / 4; ++u) {
    va[u] = __ldg(reinterpret_cast<const float4*>(pm) + u);
    vc[u] = __ldg(reinterpret_cast<const float4*>(ps) + u);
  }
  float mm = 0.f, ms = 0.f;
#pragma unroll
  for (int u = 0; u < GC::CQ / 4; ++u) {
    mm = fmaxf(mm, fmaxf(fmaxf(fabsf(va[u].x), fabsf(va[u].y)), fmaxf(fabsf(va[u].z), fabsf(va[u].w))));
    ms = fmaxf(ms, fmaxf(fmaxf(fabsf(vc[u].x), fabsf(vc[u].y)), fmaxf(fabsf(vc[u].z), fabsf(vc[u].w))));
  }
  mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, 1));
  mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, 2));
  ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, 1));
  ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, 2));
  const float scm = mm > 0.f ? kFix / mm : 0.f, scs = ms > 0.f ? kFix / ms : 0.f;
  auto digit = [&](int v) -> uint32_t {
    const int hi = (v + 128) >> 8;
    return (uint32_t)(uint8_t)(lo ? v - (hi << 8) : hi);
  };
  int ssum = 0;
#pragma unroll
  for (int u = 0; u < GC::NS; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 a = va[2 * u + h], c = vc[2 * u + h];
      const float xa[4] = {a.x, a.y, a.z, a.w}, xc[4] = {c.x, c.y, c.z, c.w};
      uint32_t dm = 0, ds = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int vmj = __float2int_rn(xa[t] * scm);
        const int vsj = __float2int_rn(xc[t] * scs);
        dm |= digit(vmj) << (8 * t);
        ds |= digit(vsj) << (8 * t);
        ssum += vsj;
      }
      f.bm[u][h] = dm;
      f.bs[u][h] = ds;
    }
  }
  // sum over the head's coordinates: the four threads of a quad hold head g/2; the
  // accumulator head of this thread is l, held by quad 2l
  ssum += __shfl_xor_sync(0xffffffffu, ssum, 1);
  ssum += __shfl_xor_sync(0xffffffffu, ssum, 2);
  ssum = __shfl_sync(0xffffffffu, ssum, 8 * l);
  mm = __shfl_sync(0xffffffffu, mm, 8 * l);
  ms = __shfl_sync(0xffffffffu, ms, 8 * l);
  f.inv_m = mm / kFix;
  f.inv_s = ms / kFix;
  f.sum_s = (float)ssum;
}

// One group's key codes of the tile's two token rows (g, g+8) and their norms.
template <class GC>
struct KeyTile {
  Words<GC::DG, GC::PK> a, b;
  float na, nb, ra, rb;
};
template <class GC>
struct ValTile {
  Words<GC::DG, GC::PV> a, b;
  float na, nb;
};

__device__ __forceinline__ float h2f(unsigned short h) { return __half2float(__ushort_as_half(h)); }

// MSE + QJL logits of one group for tokens (g, g+8) of a tile, head l.
template <class GC>
__device__ __forceinline__ void group_logits(const QOps<GC>& q, const Luts& t, const KeyTile<GC>& k, float coef,
                                             float kc_inv, float& la, float& lb) {
  int dh[4] = {0, 0, 0, 0}, dl[4] = {0, 0, 0, 0}, ds[4] = {0, 0, 0, 0};
#pragma unroll
  for (int u = 0; u < GC::NS; ++u) {
    const uint32_t sa = low_sel(k.a, u), sb = low_sel(k.b, u);
    const uint32_t sa1 = sa >> 16, sb1 = sb >> 16;
    mma_s8(dh, prmt(t.kh[0], t.kh[1], sa), prmt(t.kh[0], t.kh[1], sb), prmt(t.kh[0], t.kh[1], sa1),
           prmt(t.kh[0], t.kh[1], sb1), q.bm[u][0], q.bm[u][1]);
    mma_s8(dl, prmt(t.kl[0], t.kl[1], sa), prmt(t.kl[0], t.kl[1], sb), prmt(t.kl[0], t.kl[1], sa1),
           prmt(t.kl[0], t.kl[1], sb1), q.bm[u][0], q.bm[u][1]);
    mma_s8(ds, msb_bytes(top_bits(k.a, u, 0)), msb_bytes(top_bits(k.b, u, 0)), msb_bytes(top_bits(k.a, u, 1)),
           msb_bytes(top_bits(k.b, u, 1)), q.bs[u][0], q.bs[u][1]);
  }
  // columns 2l (query hi digit), 2l+1 (lo digit); rows g (d[0..1]) and g+8 (d[2..3])
  const float cm = kc_inv * q.inv_m;
  auto logit = [&](int i, float n, float r) {
    const float mse = fmaf(65536.f, (float)dh[i], (float)(256 * (dh[i + 1] + dl[i]) + dl[i + 1])) * cm;
    // sum_j s_j Q^_j = -2 sum_j a_j Q^_j - sum_j Q^_j  (a_j = -1 where the sign bit is set)
    const float sq = (-2.f * (float)(256 * ds[i] + ds[i + 1]) - q.sum_s) * q.inv_s;
    return n * fmaf(coef * r, sq, mse);
  };
  la += logit(0, k.na, k.ra);
  lb += logit(2, k.nb, k.rb);
}

// Value accumulation of one group: acc[u][h] (rows: the 16 coordinates 8u + 4h + t of the
// four threads of a row quad, cols: [P_hi | P_lo] heads).
template <class GC>
__device__ __forceinline__ void group_values(const Luts& t, const ValTile<GC>& v, uint32_t pb0, uint32_t pb1,
                                             float (&acc)[GC::NS][2][4]) {
#pragma unroll
  for (int u = 0; u < GC::NS; ++u) {
    const uint32_t sa = low_sel(v.a, u), sb = low_sel(v.b, u);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t xa = h ? sa >> 16 : sa, xb = h ? sb >> 16 : sb;
      const uint32_t la = prmt(t.vlo[0], t.vlo[1], xa), lb = prmt(t.vlo[0], t.vlo[1], xb);
      const uint32_t ha = prmt(t.vhi[0], t.vhi[1], xa) ^ (top_bits(v.a, u, h) & 0x80808080u);
      const uint32_t hb = prmt(t.vhi[0], t.vhi[1], xb) ^ (top_bits(v.b, u, h) & 0x80808080u);
      // token g: coordinates (4h, 4h+1) and (4h+2, 4h+3); token g+8 likewise
      const uint32_t a01 = prmt(la, ha, 0x5140u), a23 = prmt(la, ha, 0x7362u);
      const uint32_t b01 = prmt(lb, hb, 0x5140u), b23 = prmt(lb, hb, 0x7362u);
      mma16816(acc[u][h], movT(a01), movT(a23), movT(b01), movT(b23), pb0, pb1);
    }
  }
}

constexpr int kStageTok = kWarps * 16;  // tokens per pipeline stage: one 16-token tile per consumer warp
#ifndef TQ_DECODE_STAGES
#define TQ_DECODE_STAGES 4
#endif
constexpr int kNStage = TQ_DECODE_STAGES;
constexpr int kAccBytes = kWarps * kRep * 256 * 4;   // the warps' value accumulators at the end (aliases the ring)
constexpr uint64_t kDecWaitNs = 2000000000ull;
// The producer waits most of the time (the ring is full while the consumers work): its
// retries sleep instead of spinning, which leaves the issue slots to the consumer warps.
constexpr uint32_t kDecSleepNs = 2000;
#ifndef TQ_DECODE_CONSUMER_SLEEP
#define TQ_DECODE_CONSUMER_SLEEP 1
#endif

// Shared-memory layout of one pipeline stage: per group the K and V code bytes and the
// three fp16 norm arrays (key norm, residual norm, value norm) of 64 consecutive slots,
// each copied with 16-byte granularity (hence 32 bytes of slack per array).
template <class G0, class G1c, bool TWO>
struct Stage {
  static constexpr int KB0 = G0::KB, VB0 = G0::VB;
  static constexpr int KB1 = G1c::KB, VB1 = G1c::VB;
  static constexpr int NB = kStageTok * 2 + 32;                            // one norm array
  static constexpr int OFF_K0 = 0;
  static constexpr int OFF_V0 = OFF_K0 + kStageTok * KB0 + 32;
  static constexpr int OFF_K1 = OFF_V0 + kStageTok * VB0 + 32;
  static constexpr int OFF_V1 = OFF_K1 + (TWO ? kStageTok * KB1 + 32 : 0);
  static constexpr int OFF_N = OFF_V1 + (TWO ? kStageTok * VB1 + 32 : 0);   // [G][3] arrays of NB bytes
  static constexpr int BYTES = ((OFF_N + (TWO ? 2 : 1) * 3 * NB) + 127) / 128 * 128;
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
__global__ void __launch_bounds__((kWarps + 1) * 32, TQ_DECODE_CTAS_PER_SM) decode_mma_kernel(MmaArgs A) {
  constexpr bool TWO = !std::is_same<G1, void>::value;
  constexpr int NG = TWO ? 2 : 1;
  using G1c = typename std::conditional<TWO, G1, G0>::type;
  using ST = Stage<G0, G1c, TWO>;
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ float s_m[kWarps][kRep], s_l[kWarps][kRep];
  float(*s_acc)[kRep][256] = reinterpret_cast<float(*)[kRep][256]>(dsm);   // used once the ring is drained
  __shared__ __align__(8) uint64_t full[kNStage], empty[kNStage];
  __shared__ int s_abort;
  const int split = blockIdx.x, bh = blockIdx.y / A.nsub, sub = blockIdx.y % A.nsub;
  const int b = bh / A.Hkv, hk = bh % A.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int T = max(0, (int)min((int64_t)A.seq_lens[b], A.max_len));
  const int t_begin = split * A.chunk;
  const int t_end = min(T, t_begin + A.chunk);
  const int64_t slot0 = (int64_t)bh * A.max_len;
  // The merge kernel behind this one may launch once every CTA of this grid has run this
  // trigger (or exited), so its CTAs only take slots of the last wave; its grid-dependency
  // wait still waits for the whole grid, so it sees every partial.
  allow_dependent_launch();
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

  // ------------------------------------------------------------------ consumer warps
  // (their code comes first: the consumers' path from the kernel entry is straight-line,
  // which shortens the cold instruction fetch before their first loads)
  float acc0[G0::NS][2][4];
  float acc1[G1c::NS][2][4];
  float m_run = -INFINITY, l_run = 0.f;
  if (warp < kWarps) {
    const Luts t0 = A.g[0].lut;
    const Luts t1 = A.g[TWO ? 1 : 0].lut;
    grid_dependency_wait();   // prepared queries come from the preceding kernel
    QOps<G0> q0;
    load_qops<G0>(q0, A, 0, b, hk, sub, lane);
    QOps<G1c> q1;
    if constexpr (TWO) load_qops<G1c>(q1, A, 1, b, hk, sub, lane);
#pragma unroll
    for (int u = 0; u < G0::NS; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h) acc0[u][h][0] = acc0[u][h][1] = acc0[u][h][2] = acc0[u][h][3] = 0.f;
#pragma unroll
    for (int u = 0; u < G1c::NS; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h) acc1[u][h][0] = acc1[u][h][1] = acc1[u][h][2] = acc1[u][h][3] = 0.f;
    int it = 0;
    // Where a staged array's first slot lands inside its stage buffer: the bulk copies keep
    // the source's offset within 16 bytes.  Stages start at multiples of 64 tokens (and
    // pages hold multiples of 64 slots), so the offset is the same for every stage.
    const int64_t sbase = A.table ? 0 : slot0;
    const int ja = warp * 16 + g, jb = ja + 8;   // stage-local token rows of this lane
    const int ok0 = (int)((sbase * ST::KB0) & 15) + ST::OFF_K0, ov0 = (int)((sbase * ST::VB0) & 15) + ST::OFF_V0;
    const int ok1 = (int)((sbase * ST::KB1) & 15) + ST::OFF_K1, ov1 = (int)((sbase * ST::VB1) & 15) + ST::OFF_V1;
    const int nof = (int)((sbase * 2) & 15) + ST::OFF_N;
    for (int ts = t_begin; ts < t_end; ts += kStageTok, ++it) {
      const int s = it % kNStage;
#if TQ_DECODE_CONSUMER_SLEEP
      if (!mbar_wait_sleep(full + s, (it / kNStage) & 1, abort_v, kDecWaitNs, kDecSleepNs)) { fail(202); break; }
#else
      if (!mbar_wait(full + s, (it / kNStage) & 1, abort_v, kDecWaitNs)) { fail(202); break; }
#endif
      const int tt = ts + warp * 16;           // this warp's 16-token tile
      const bool live = tt < t_end;
      const uint8_t* st = dsm + s * ST::BYTES;
      KeyTile<G0> k0;
      ValTile<G0> v0;
      KeyTile<G1c> k1;
      ValTile<G1c> v1;
      if (live) {
        lds_words(k0.a, st + ok0 + ja * ST::KB0, l);
        lds_words(k0.b, st + ok0 + jb * ST::KB0, l);
        lds_words(v0.a, st + ov0 + ja * ST::VB0, l);
        lds_words(v0.b, st + ov0 + jb * ST::VB0, l);
        // value norms of slots past the context (staged bytes of other slots, or bytes never
        // written) read as 0; key norms need no guard, those tokens' logits become -inf
        const bool va = tt + g < t_end, vb = tt + g + 8 < t_end;
        auto nrm = [&](int gi, int a, int j) {
          return h2f(reinterpret_cast<const uint16_t*>(st + nof + (gi * 3 + a) * ST::NB)[j]);
        };
        k0.na = nrm(0, 0, ja); k0.nb = nrm(0, 0, jb);
        k0.ra = nrm(0, 1, ja); k0.rb = nrm(0, 1, jb);
        v0.na = va ? nrm(0, 2, ja) : 0.f; v0.nb = vb ? nrm(0, 2, jb) : 0.f;
        if constexpr (TWO) {
          lds_words(k1.a, st + ok1 + ja * ST::KB1, l);
          lds_words(k1.b, st + ok1 + jb * ST::KB1, l);
          lds_words(v1.a, st + ov1 + ja * ST::VB1, l);
          lds_words(v1.b, st + ov1 + jb * ST::VB1, l);
          k1.na = nrm(1, 0, ja); k1.nb = nrm(1, 0, jb);
          k1.ra = nrm(1, 1, ja); k1.rb = nrm(1, 1, jb);
          v1.na = va ? nrm(1, 2, ja) : 0.f; v1.nb = vb ? nrm(1, 2, jb) : 0.f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);   // the stage's data now sits in registers
      if (!live) continue;
      float la = 0.f, lb = 0.f;
      group_logits<G0>(q0, t0, k0, A.g[0].coef, A.g[0].kc_inv, la, lb);
      if constexpr (TWO) group_logits<G1c>(q1, t1, k1, A.g[1].coef, A.g[1].kc_inv, la, lb);
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
        for (int u = 0; u < G0::NS; ++u)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc0[u][h][i] *= alpha;
        if constexpr (TWO) {
#pragma unroll
          for (int u = 0; u < G1c::NS; ++u)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int i = 0; i < 4; ++i) acc1[u][h][i] *= alpha;
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
      pfrag(v0.na, v0.nb, pb0, pb1);
      group_values<G0>(t0, v0, pb0, pb1, acc0);
      if constexpr (TWO) {
        pfrag(v1.na, v1.nb, pb0, pb1);
        group_values<G1c>(t1, v1, pb0, pb1, acc1);
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
  } else {
    // ---------------------------------------------------------------- producer warp
    if (split == 0 && blockIdx.y == 0 && lane < (TWO ? 2 : 1)) bulk_prefetch_l2(A.piv[lane], A.piv_bytes[lane]);
    int it = 0;
    uint32_t issued = 0, phases = 0;           // stages with copies issued, parity of their last phase
    for (int ts = t_begin; ts < t_end; ts += kStageTok, ++it) {
      const int s = it % kNStage;
      const uint32_t ph = (it / kNStage) & 1;
      if (!mbar_wait_sleep(empty + s, ph ^ 1, abort_v, kDecWaitNs, kDecSleepNs)) { fail(201); break; }
      const int ntok = min(kStageTok, t_end - ts);
      uint8_t* st = dsm + s * ST::BYTES;
      const int64_t first = stage_slot(A, b, hk, ts, slot0), last = first + ntok;
      // one array per lane: lanes 0..2NG-1 the code arrays (K0, V0[, K1, V1]), the next 3NG
      // lanes the norm arrays (key norm, residual norm, value norm of each group); each lane
      // adds its own bytes to the stage's transaction count before its copy
      if (lane < 5 * NG) {
        const bool nrm = lane >= 2 * NG;
        const int j = nrm ? lane - 2 * NG : lane;
        const int gi = TWO ? (nrm ? j / 3 : j >> 1) : 0;
        const int kind = nrm ? j % 3 : (j & 1);            // codes: 0 K, 1 V; norms: 0 kn, 1 kr, 2 vn
        const MmaGroup& gr = A.g[0];
        const MmaGroup& gq = A.g[TWO ? 1 : 0];
        const bool second = gi != 0;
        const uint8_t* src;
        int64_t eb, cap;
        int doff;
        if (!nrm) {
          const bool v = kind != 0;
          src = v ? (second ? gq.vcodes : gr.vcodes) : (second ? gq.kcodes : gr.kcodes);
          eb = v ? (second ? ST::VB1 : ST::VB0) : (second ? ST::KB1 : ST::KB0);
          cap = v ? (second ? gq.vcap : gr.vcap) : (second ? gq.kcap : gr.kcap);
          doff = v ? (second ? ST::OFF_V1 : ST::OFF_V0) : (second ? ST::OFF_K1 : ST::OFF_K0);
        } else {
          const uint16_t* p = kind == 0 ? (second ? gq.knorm : gr.knorm)
                                        : kind == 1 ? (second ? gq.krnorm : gr.krnorm) : (second ? gq.vnorm : gr.vnorm);
          src = reinterpret_cast<const uint8_t*>(p);
          eb = 2;
          cap = kind < 2 ? (second ? gq.kcap : gr.kcap) : (second ? gq.vcap : gr.vcap);
          doff = ST::OFF_N + (gi * 3 + kind) * ST::NB;
        }
        const uint32_t bytes = stage_span(st + doff, src, first * eb, last * eb, cap * eb, full + s, false);
        if (bytes) mbar_expect_tx(full + s, bytes);
        stage_span(st + doff, src, first * eb, last * eb, cap * eb, full + s, true);
      }
      __syncwarp();
      mbar_arrive(full + s);
      issued |= 1u << s;
      phases = (phases & ~(1u << s)) | (ph << s);
    }
    // bulk copies still in flight land before the CTA exits
    if (lane == 0)
      for (int i = 0; i < kNStage; ++i)
        if ((issued >> i) & 1u) mbar_wait(full + i, (phases >> i) & 1u, nullptr, kDecWaitNs);
    __syncwarp();
  }
  __syncthreads();   // the ring is drained: its memory now holds the warps' accumulators
  if (warp < kWarps) {
    // row g of block (u, h) is coordinate CQ (g>>1) + 8u + 4h + (g&1), row g+8 adds 2
    auto store_acc = [&](auto& acc, auto gc_tag, int off) {
      using GC = decltype(gc_tag);
#pragma unroll
      for (int u = 0; u < GC::NS; ++u)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = GC::CQ * (g >> 1) + 8 * u + 4 * h + (g & 1);
          s_acc[warp][l][off + c] = acc[u][h][0] + acc[u][h][1];
          s_acc[warp][l][off + c + 2] = acc[u][h][2] + acc[u][h][3];
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
    if (sub * kRep + h >= A.rep) continue;       // a repeated column: not one of this kv head's heads
    float* dst = A.part + (size_t)(b * A.Hq + hk * A.rep + sub * kRep + h) * A.part_ld + (size_t)split * (A.D + 2);
    if (c == 0) {
      dst[0] = (M == -INFINITY) ? -INFINITY : M * ln2;
      dst[1] = L;
    }
    dst[2 + c] = acc;
  }
}

// Rotated queries Pi q and S q of every group in fp32 (the fixed-point digits are formed by
// the consumer warps of the decode kernel, which see a whole head row), one launch for all
// groups.  CTA = 16 query rows x 16 outputs of one (group, part): the 16 columns of Pi^T
// (part 0) or S^T (part 1) and the 16 rows (channels gathered through the permutation) are
// staged in shared memory with one round of loads; thread (row, 4 outputs, K quarter) runs
// 4 dot products over a quarter of the d_g terms and the quarters are summed by shuffles.  The decode kernel is launched behind it and starts streaming the
// cache at once; its consumer warps wait for this grid before reading the projections.
constexpr int kPrepRows = 16;

struct PrepArgs {
  const void* q;
  int q_f32;
  int nrows, D, G, Hq, rep, dg, obs;   // obs: output blocks (16 or 64 outputs) per group
  const int32_t* perm;                 // [Hkv][D] channel permutation or NULL
  int off[2];
  const float* pit[2];
  const float* stt[2];
  float* qp;                           // [nrows][G][2][D]
};

__global__ void __launch_bounds__(256) decode_prep_kernel(PrepArgs A) {
  __shared__ __align__(16) float ms[128][16];        // [j][o]: M^T[j][16 ob + o]
  __shared__ float xs[kPrepRows][129];               // padded rows
  allow_dependent_launch();
  const int r0 = blockIdx.x * kPrepRows;
  const int y = blockIdx.y;                          // (group, part, 16-output block)
  const int ob = y % A.obs, part = (y / A.obs) & 1, gi = y / (2 * A.obs);
  const int dg = A.dg, t = threadIdx.x;
  const float* M = gi ? (part ? A.stt[1] : A.pit[1]) : (part ? A.stt[0] : A.pit[0]);
  const int off = gi ? A.off[1] : A.off[0];
  for (int e = t; e < dg * 4; e += 256) {
    const int jj = e >> 2, c4 = e & 3;
    *reinterpret_cast<float4*>(&ms[jj][4 * c4]) =
        __ldg(reinterpret_cast<const float4*>(M + (size_t)jj * dg + 16 * ob) + c4);
  }
  for (int e = t; e < kPrepRows * dg; e += 256) {
    const int r = e / dg, jj = e % dg;
    float v = 0.f;
    if (r0 + r < A.nrows) {
      const size_t row = (size_t)(r0 + r) * A.D;
      int ch = off + jj;
      if (A.perm) ch = __ldg(A.perm + (size_t)(((r0 + r) % A.Hq) / A.rep) * A.D + off + jj);
      if (ch >= 0 && ch < A.D)   // (the merge kernel reports an out-of-range entry)
        v = A.q_f32 ? __ldg(static_cast<const float*>(A.q) + row + ch)
                    : __bfloat162float(static_cast<const __nv_bfloat16*>(A.q)[row + ch]);
    }
    xs[r][jj] = v;
  }
  __syncthreads();
  // thread = (row, 4-output group, K quarter): terms j = 4 i + kq, then the four quarters
  // (adjacent lanes) are summed by shuffles
  const int kq = t & 3, og = (t >> 2) & 3, r = t >> 4;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int jj = kq; jj < dg; jj += 4) {
    const float4 m = *reinterpret_cast<const float4*>(&ms[jj][4 * og]);
    const float x = xs[r][jj];
    a[0] = fmaf(m.x, x, a[0]);
    a[1] = fmaf(m.y, x, a[1]);
    a[2] = fmaf(m.z, x, a[2]);
    a[3] = fmaf(m.w, x, a[3]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    a[k] += __shfl_xor_sync(0xffffffffu, a[k], 1);
    a[k] += __shfl_xor_sync(0xffffffffu, a[k], 2);
  }
  if (kq == 0 && r0 + r < A.nrows)
    *reinterpret_cast<float4*>(A.qp + ((size_t)(r0 + r) * A.G + gi) * 2 * A.D + part * A.D + 16 * ob + 4 * og) =
        make_float4(a[0], a[1], a[2], a[3]);
}

// The same projection for many query rows: CTA = 16 rows x 64 outputs, thread = (row, 4
// outputs) over all d_g terms; four times fewer CTAs than the 16-output form, so that a
// large batch's prep leaves the SMs to the decode kernel sooner.
__global__ void __launch_bounds__(256) decode_prep_wide_kernel(PrepArgs A) {
  __shared__ __align__(16) float ms[128][64];        // [j][o]: M^T[j][64 ob + o]
  __shared__ float xs[kPrepRows][129];               // padded rows: conflict-free reads
  allow_dependent_launch();
  const int r0 = blockIdx.x * kPrepRows;
  const int y = blockIdx.y;                          // (group, part, output block)
  const int ob = y % A.obs, part = (y / A.obs) & 1, gi = y / (2 * A.obs);
  const int dg = A.dg, t = threadIdx.x;
  const float* M = gi ? (part ? A.stt[1] : A.pit[1]) : (part ? A.stt[0] : A.pit[0]);
  const int off = gi ? A.off[1] : A.off[0];
  for (int e = t; e < dg * 16; e += 256) {
    const int j = e >> 4, c4 = e & 15;
    *reinterpret_cast<float4*>(&ms[j][4 * c4]) =
        __ldg(reinterpret_cast<const float4*>(M + (size_t)j * dg + 64 * ob) + c4);
  }
  for (int e = t; e < kPrepRows * dg; e += 256) {
    const int r = e / dg, j = e % dg;
    float v = 0.f;
    if (r0 + r < A.nrows) {
      const size_t row = (size_t)(r0 + r) * A.D;
      int ch = off + j;
      if (A.perm) ch = __ldg(A.perm + (size_t)(((r0 + r) % A.Hq) / A.rep) * A.D + off + j);
      if (ch >= 0 && ch < A.D)   // (the merge kernel reports an out-of-range entry)
        v = A.q_f32 ? __ldg(static_cast<const float*>(A.q) + row + ch)
                    : __bfloat162float(static_cast<const __nv_bfloat16*>(A.q)[row + ch]);
    }
    xs[r][j] = v;
  }
  __syncthreads();
  const int r = t % kPrepRows, og = t / kPrepRows;   // row, output group (4 outputs)
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int j = 0; j < dg; ++j) {
    const float4 m = *reinterpret_cast<const float4*>(&ms[j][4 * og]);
    const float x = xs[r][j];
    a[0] = fmaf(m.x, x, a[0]);
    a[1] = fmaf(m.y, x, a[1]);
    a[2] = fmaf(m.z, x, a[2]);
    a[3] = fmaf(m.w, x, a[3]);
  }
  if (r0 + r < A.nrows)
    *reinterpret_cast<float4*>(A.qp + ((size_t)(r0 + r) * A.G + gi) * 2 * A.D + part * A.D + 64 * ob + 4 * og) =
        make_float4(a[0], a[1], a[2], a[3]);
}

// Arguments of the merge kernel (below).
struct Merge2Args {
  const float* part;
  int64_t part_ld;
  int nsplit, D, G;
  int off[3];
  const float* PiV[2];
  float* out;
  const int32_t* perm;   // channel permutation [Hkv][D] (NULL: identity): group channel c -> perm[kv][c]
  int Hq, rep, Hkv, nsub;
  int pi_floats;         // floats of the staged rotations (a multiple of 4)
  int stage_parts;       // copy the CTA's split partials into shared memory first (they fit)
  int* err;
};

// Log-sum-exp merge of the context splits and the inverse value rotation, one CTA per
// (sequence, kv head, group of 4 query heads): thread (head, coordinate) folds the splits'
// (m, l, acc) against the maximum taken in a first pass, the merged rotated values go
// to shared memory, and thread (output channel) applies the group's Pi_v^T to all 4 heads
// with one read of every rotation entry (the rotation is read once per CTA, not once per
// query row and channel block).
constexpr int kMergeHThreads = 256;
constexpr int kMergeMaxSplit = 512;       // the split count is at most this (checked at launch)

__global__ void __launch_bounds__(kMergeHThreads, 4) decode_merge_heads_kernel(Merge2Args A) {
  extern __shared__ __align__(16) float s_pi[];   // the value groups' Pi, [dg0^2 | dg1^2] (row-major)
  __shared__ float s_v[kRep][256];                // merged rotated values (<= 256 channels)
  __shared__ float s_w[kRep][kMergeMaxSplit];     // per head and split: e^(m_s - M)
  __shared__ float s_red[kRep][2][2];             // per head: the two warps' maxima, then their sums
  const int D = A.D, ns = A.nsplit, W = D + 2;
  const int bh = blockIdx.x / A.nsub, sub = blockIdx.x % A.nsub;
  const int b = bh / A.Hkv, hk = bh % A.Hkv;
  const int nh = min(kRep, A.rep - sub * kRep);      // query heads of this CTA
  const int row0 = b * A.Hq + hk * A.rep + sub * kRep;
  const int h = threadIdx.x >> 6, t64 = threadIdx.x & 63;   // head, lane of the head
  const int wh = (threadIdx.x >> 5) & 1;                     // warp of the head
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    s_ok = 1;
    fence_barrier_init();
  }
  // the rotations are constant: staged while the decode grid still runs
  {
    const int n0 = (A.off[1] - A.off[0]) * (A.off[1] - A.off[0]);
    const int n1 = A.G > 1 ? (A.off[2] - A.off[1]) * (A.off[2] - A.off[1]) : 0;
    for (int e = 4 * threadIdx.x; e < n0 + n1; e += 4 * kMergeHThreads) {
      const float* src = e < n0 ? A.PiV[0] + e : A.PiV[1] + (e - n0);
      *reinterpret_cast<float4*>(s_pi + e) = __ldg(reinterpret_cast<const float4*>(src));
    }
  }
  __syncthreads();
  grid_dependency_wait();    // every partial of the decode grid is written
  // With few splits the CTA's partial rows (nh rows of part_ld floats, 16-byte multiples)
  // come into shared memory by bulk copies in one round trip; the passes below then read
  // shared memory instead of making a dependent global round trip per split.
  float* s_parts = s_pi + A.pi_floats;
  if (A.stage_parts) {
    if (threadIdx.x == 0) {
      const uint32_t bytes = (uint32_t)(A.part_ld * sizeof(float));
      mbar_arrive_expect_tx(&s_bar, bytes * (uint32_t)nh);
      for (int hh = 0; hh < nh; ++hh)
        bulk_load(s_parts + (size_t)hh * A.part_ld, A.part + (size_t)(row0 + hh) * A.part_ld, bytes, &s_bar);
      if (!mbar_wait(&s_bar, 0, nullptr, kDecWaitNs)) {
        s_ok = 0;
        if (A.err) atomicCAS(A.err, 0, 203);
      }
    }
    __syncthreads();
    if (!s_ok) return;   // (every thread of the CTA leaves here)
  }
  // pass 1: the head's maximum over the splits, the weights e^(m_s - M) and L = sum_s w_s l_s
  const float* P = A.stage_parts ? s_parts + (size_t)min(h, nh - 1) * A.part_ld
                                 : A.part + (size_t)(row0 + min(h, nh - 1)) * A.part_ld;
  float mloc[kMergeMaxSplit / 64], lloc[kMergeMaxSplit / 64];
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMergeMaxSplit / 64; ++i) {
    const int s2 = t64 + 64 * i;
    mloc[i] = s2 < ns ? P[(size_t)s2 * W] : -INFINITY;
    lloc[i] = s2 < ns ? P[(size_t)s2 * W + 1] : 0.f;
    M = fmaxf(M, mloc[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((threadIdx.x & 31) == 0) s_red[h][wh][0] = M;
  __syncthreads();
  M = fmaxf(s_red[h][0][0], s_red[h][1][0]);
  float L = 0.f;
#pragma unroll
  for (int i = 0; i < kMergeMaxSplit / 64; ++i) {
    const int s2 = t64 + 64 * i;
    const float w = (mloc[i] == -INFINITY) ? 0.f : __expf(mloc[i] - M);
    if (s2 < ns) s_w[h][s2] = w;
    L = fmaf(w, lloc[i], L);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  if ((threadIdx.x & 31) == 0) s_red[h][wh][1] = L;
  __syncthreads();
  L = s_red[h][0][1] + s_red[h][1][1];
  // pass 2: the merged accumulators of the head (coordinates t64 + 64 j)
  {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int s2 = 0; s2 < ns; ++s2) {   // (8 splits' loads in flight: long split lists are latency-bound)
      const float* ps = P + (size_t)s2 * W + 2;
      const float w = s_w[h][s2];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (t64 + 64 * j < D) acc[j] = fmaf(w, ps[t64 + 64 * j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (t64 + 64 * j < D) s_v[h][t64 + 64 * j] = L > 0.f ? acc[j] / L : 0.f;
  }
  __syncthreads();
  // inverse rotation of each group: out[ch] = sum_i Pi_g[i][ch - off] v[off + i]
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const bool second = A.G > 1 && c >= A.off[1];
    const int goff = second ? A.off[1] : A.off[0], gd = (second ? A.off[2] : A.off[1]) - goff;
    const float* Pi = s_pi + (second ? (A.off[1] - A.off[0]) * (A.off[1] - A.off[0]) : 0) + (c - goff);
    float o[kRep] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int i = 0; i < gd; ++i) {
      const float pv = Pi[i * gd];
#pragma unroll
      for (int hh = 0; hh < kRep; ++hh) o[hh] = fmaf(pv, s_v[hh][goff + i], o[hh]);
    }
    const int oc_ch = A.perm ? A.perm[(size_t)hk * D + c] : c;
    if (oc_ch < 0 || oc_ch >= D) {
      if (A.err) atomicCAS(A.err, 0, (int)kErrPermRange);
      continue;
    }
#pragma unroll
    for (int hh = 0; hh < kRep; ++hh)
      if (hh < nh) A.out[(size_t)(row0 + hh) * D + oc_ch] = o[hh];
  }
}

// Rotated queries of all groups (one launch).
int launch_prep(const void* q, int q_dtype, int nrows, const tq_ctx* const* kctx, const int* off, int G, float* qp,
                int D, const int32_t* perm, int Hq, int rep, cudaStream_t st) {
  PrepArgs P{};
  P.q = q; P.q_f32 = q_dtype == TQ_DTYPE_F32; P.nrows = nrows; P.D = D; P.G = G; P.Hq = Hq; P.rep = rep;
  P.dg = kctx[0]->lay.d; P.obs = P.dg / 16; P.perm = perm; P.qp = qp;
  for (int g = 0; g < G; ++g) { P.off[g] = off[g]; P.pit[g] = kctx[g]->PiT; P.stt[g] = kctx[g]->ST; }
  if (nrows > 256) {
    P.obs = P.dg / 64;
    const dim3 grid((nrows + kPrepRows - 1) / kPrepRows, G * 2 * P.obs);
    decode_prep_wide_kernel<<<grid, 256, 0, st>>>(P);
  } else {
    const dim3 grid((nrows + kPrepRows - 1) / kPrepRows, G * 2 * P.obs);
    decode_prep_kernel<<<grid, 256, 0, st>>>(P);
  }
  count_launch();
  return check_launch("decode_prep_kernel");
}

// Words of a record from global memory (same shapes as lds_words).
template <int DG, int P>
__device__ __forceinline__ void ldg_words(Words<DG, P>& r, const uint8_t* rec, int l) {
  if constexpr (DG == 128 && P == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(rec + 16 * l));
    r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
  } else if constexpr (DG == 64 && P == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(rec + 8 * l));
    r.w[0] = v.x; r.w[1] = v.y;
  } else if constexpr (DG == 128) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(rec + 4 * P * l);
#pragma unroll
    for (int i = 0; i < P; ++i) r.w[i] = __ldg(p + i);
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(rec + 4 * P * (l >> 1));
#pragma unroll
    for (int i = 0; i < P; ++i) r.w[i] = __ldg(p + i);
    const int odd = l & 1;
    if constexpr (P == 3) {
      r.w[0] >>= 2 * odd;
      r.w[1] >>= 2 * odd;
    } else {
      r.w[0] >>= 2 * odd;
    }
    r.w[P - 1] <<= 4 * odd;
  }
}

// Standalone attention logits on the tensor cores.  A logit is compared to the float64
// definition at 1e-3 absolute, about 2^-17 of |q||k| for unit-scale d = 128 vectors, so
// this kernel carries both operands at ~2^-22: centroids as fp16 hi + lo (two A
// operands), the prepared query Pi q / S q as fp16 hi + lo in the 8 columns (4 queries x
// hi/lo), products exact in the fp32 accumulator (m16n8k16).  CTA = (key range, block of
// kRep queries), 4 warps; every warp scores 16 keys per step.
struct LogitArgs {
  const uint8_t* codes;
  const uint16_t* norm;
  const uint16_t* rnorm;
  const float* qprep;     // [nq][2d]: (Pi q, S q) in fp32
  int64_t n, keys_per_cta;
  int nq, d;
  float coef;
  uint32_t ch[2][2], cl[2][2];   // fp16 centroid tables by code: [low byte, high byte] of c_hi, c_lo
  float* out;
};

// fp16 pairs of coordinates (4h, 4h+1), (4h+2, 4h+3) of a half-slice from byte tables
__device__ __forceinline__ void lookup16(const uint32_t (&t)[2][2], uint32_t sel, uint32_t& x01, uint32_t& x23) {
  const uint32_t L = prmt(t[0][0], t[0][1], sel), H = prmt(t[1][0], t[1][1], sel);
  x01 = prmt(L, H, 0x5140u);
  x23 = prmt(L, H, 0x7362u);
}
// +-1.0 in fp16 for the same coordinates: msb of byte t of `top` set -> +1 (sign bit [S r >= 0])
__device__ __forceinline__ void signs16(uint32_t top, uint32_t& x01, uint32_t& x23) {
  const uint32_t H = (~top & 0x80808080u) | 0x3C3C3C3Cu;   // fp16 high bytes of +1 / -1
  x01 = prmt(0u, H, 0x5040u);
  x23 = prmt(0u, H, 0x7060u);
}

template <class GC>
__global__ void __launch_bounds__(128) logits_mma_kernel(LogitArgs A) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, l = lane & 3;
  const int qb = blockIdx.y;
  // B fragments: column g = query qb*kRep + g/2, hi (g even) or lo part; k-slots of
  // (slice u, half h) = this thread's coordinates CQ l + 8u + 4h + {0, 1 | 2, 3}
  uint32_t bm[GC::NS][2][2], bs[GC::NS][2][2];
  {
    const int qrow = qb * kRep + (g >> 1);
    const bool lo = (g & 1) != 0;
    const float* src = A.qprep + (size_t)(qrow < A.nq ? qrow : 0) * 2 * A.d;
    const bool ok = qrow < A.nq;
    auto part = [&](float v) {
      if (!ok) return 0.f;
      const float h = __half2float(__float2half_rn(v));
      return lo ? v - h : h;
    };
    // the thread's coordinates come four at a time (16-byte loads: d and 2d are multiples
    // of 4, and each group of four starts at a multiple of 4)
#pragma unroll
    for (int u = 0; u < GC::NS; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = GC::CQ * l + 8 * u + 4 * h;
        const float4 vm = __ldg(reinterpret_cast<const float4*>(src + c));
        const float4 vs = __ldg(reinterpret_cast<const float4*>(src + A.d + c));
        bm[u][h][0] = pack_h2(part(vm.x), part(vm.y));
        bm[u][h][1] = pack_h2(part(vm.z), part(vm.w));
        bs[u][h][0] = pack_h2(part(vs.x), part(vs.y));
        bs[u][h][1] = pack_h2(part(vs.z), part(vs.w));
      }
  }
  const int64_t k0 = (int64_t)blockIdx.x * A.keys_per_cta;
  const int64_t k1 = min(A.n, k0 + A.keys_per_cta);
  const int qi = qb * kRep + l;
  // code words and norms of a warp's 16-key tiles are loaded three steps ahead of their
  // use, so the global-memory latency overlaps the tensor-core work
  struct Tile {
    Words<GC::DG, GC::PK> wa, wb;
    float na, ra, nb, rb;
  };
  auto load = [&](int64_t base, Tile& T) {
    const int64_t ka = base + g, kb = base + g + 8;
    const bool va = ka < k1, vb = kb < k1;
#pragma unroll
    for (int i = 0; i < Words<GC::DG, GC::PK>::N; ++i) T.wa.w[i] = T.wb.w[i] = 0u;
    if (va) ldg_words(T.wa, A.codes + ka * GC::KB, l);
    if (vb) ldg_words(T.wb, A.codes + kb * GC::KB, l);
    T.na = va ? h2f(__ldg(A.norm + ka)) : 0.f;
    T.ra = va ? h2f(__ldg(A.rnorm + ka)) : 0.f;
    T.nb = vb ? h2f(__ldg(A.norm + kb)) : 0.f;
    T.rb = vb ? h2f(__ldg(A.rnorm + kb)) : 0.f;
  };
  auto compute = [&](const Tile& cur, int64_t base) {
    const int64_t ka = base + g, kb = base + g + 8;
    const bool va = ka < k1, vb = kb < k1;
    float mse[4] = {0.f, 0.f, 0.f, 0.f}, sgn[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < GC::NS; ++u) {
      const uint32_t sa = low_sel(cur.wa, u), sb = low_sel(cur.wb, u);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t xa = h ? sa >> 16 : sa, xb = h ? sb >> 16 : sb;
        uint32_t a01, a23, b01, b23;
        lookup16(A.ch, xa, a01, a23);
        lookup16(A.ch, xb, b01, b23);
        mma16816(mse, a01, b01, a23, b23, bm[u][h][0], bm[u][h][1]);
        lookup16(A.cl, xa, a01, a23);
        lookup16(A.cl, xb, b01, b23);
        mma16816(mse, a01, b01, a23, b23, bm[u][h][0], bm[u][h][1]);
        signs16(top_bits(cur.wa, u, h), a01, a23);
        signs16(top_bits(cur.wb, u, h), b01, b23);
        mma16816(sgn, a01, b01, a23, b23, bs[u][h][0], bs[u][h][1]);
      }
    }
    const float la = cur.na * fmaf(A.coef * cur.ra, sgn[0] + sgn[1], mse[0] + mse[1]);
    const float lb = cur.nb * fmaf(A.coef * cur.rb, sgn[2] + sgn[3], mse[2] + mse[3]);
    if (qi < A.nq) {
      if (va) A.out[(size_t)qi * A.n + ka] = la;
      if (vb) A.out[(size_t)qi * A.n + kb] = lb;
    }
  };
  // three 16-key tiles of this warp in flight: the tile three steps ahead is requested as
  // soon as a tile's registers are free
  Tile t0, t1, t2;
  const int64_t b0 = k0 + warp * 16;
  if (b0 < k1) load(b0, t0);
  if (b0 + 64 < k1) load(b0 + 64, t1);
  if (b0 + 128 < k1) load(b0 + 128, t2);
  for (int64_t base = b0; base < k1; base += 192) {
    compute(t0, base);
    if (base + 192 < k1) load(base + 192, t0);
    if (base + 64 >= k1) break;
    compute(t1, base + 64);
    if (base + 256 < k1) load(base + 256, t1);
    if (base + 128 >= k1) break;
    compute(t2, base + 128);
    if (base + 320 < k1) load(base + 320, t2);
  }
}

template <class GC>
int launch_logits_t(LogitArgs A, cudaStream_t st) {
  const int nqb = (A.nq + kRep - 1) / kRep;
  // about 4 CTAs per SM in total, one wave (the query fragments are built once per CTA),
  // whole 64-key steps per CTA
  int64_t ctas = (int64_t)148 * 4 / nqb;
  if (ctas < 1) ctas = 1;
  int64_t per = (A.n + ctas - 1) / ctas;
  per = ((per + 63) / 64) * 64;
  if (per < 64) per = 64;
  A.keys_per_cta = per;
  const int64_t nblk = (A.n + per - 1) / per;
  logits_mma_kernel<GC><<<dim3((unsigned)nblk, (unsigned)nqb), 128, 0, st>>>(A);
  count_launch();
  return check_launch("logits_mma_kernel");
}

template <class G0, class G1>
int launch_mma_t(const MmaArgs& A, int nsplit, int BHkv, cudaStream_t st) {
  constexpr bool TWO = !std::is_same<G1, void>::value;
  using G1c = typename std::conditional<TWO, G1, G0>::type;
  const int dyn = std::max(kNStage * Stage<G0, G1c, TWO>::BYTES, kAccBytes);
  // one shared-memory carveout for the prep, decode and merge kernels, so they can share SMs
  cudaError_t ea = ensure_smem_attrs<decode_mma_kernel<G0, G1>>(dyn, true);
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

int decode_mma_ctas_per_sm() { return TQ_DECODE_CTAS_PER_SM; }

// Tables of one (key context, value context) pair; returns the key-centroid scale inverse.
float mmaops::host_luts(const tq_ctx* kc, const tq_ctx* vc, Luts* t) {
  *t = Luts{};
  const Codebook& kb = kc->cb;
  float cmax = 0.f;
  for (int j = 0; j < kb.K; ++j) cmax = fmaxf(cmax, fabsf(kb.c[j]));
  const float sc = cmax > 0.f ? kFix / cmax : 0.f;
  for (int code = 0; code < kb.K && code < 8; ++code) {
    const int C = (int)lrintf(kb.cc[code] * sc);
    const int hi = (C + 128) >> 8, lo = C - (hi << 8);
    t->kh[code / 4] |= (uint32_t)(uint8_t)hi << (8 * (code % 4));
    t->kl[code / 4] |= (uint32_t)(uint8_t)lo << (8 * (code % 4));
  }
  const Codebook& vb = vc->cb;
  const int half = vb.K / 2;
  for (int m = 0; m < half && m < 8; ++m) {
    __half hv = __float2half_rn(vb.c[half + m]);
    const uint16_t bits = *reinterpret_cast<uint16_t*>(&hv);
    t->vlo[m / 4] |= (uint32_t)(bits & 0xFF) << (8 * (m % 4));
    t->vhi[m / 4] |= (uint32_t)(bits >> 8) << (8 * (m % 4));
  }
  return sc > 0.f ? 1.f / sc : 0.f;
}

// Returns kNotHandled when the shape is outside this kernel's instantiations.
int launch_decode_mma(const tq_ctx* const* kctx, const tq_ctx* const* vctx, const int* off, int G,
                      const int32_t* perm, const int32_t* table, int page, const void* q, int q_dtype,
                      const tq_packed* kc, const tq_packed* vc, const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                      int64_t max_len, float scale, float* out, void* ws, cudaStream_t st) {
  if (G > 2 || D > 256) return kNotHandled;
  int sig[2] = {0, 0};
  for (int g = 0; g < G; ++g) {
    const int dg = kctx[g]->lay.d;
    if (dg != 64 && dg != 128) return kNotHandled;
    sig[g] = dg * 100 + kctx[g]->lay.planes * 10 + vctx[g]->lay.planes;
  }
  auto is = [&](int a, int bsig) { return sig[0] == a && sig[1] == bsig; };
  using C128_44 = GroupCfg<128, 4, 4>;
  using C128_33 = GroupCfg<128, 3, 3>;
  using C64_44 = GroupCfg<64, 4, 4>;
  using C64_33 = GroupCfg<64, 3, 3>;
  using C64_22 = GroupCfg<64, 2, 2>;
  const bool ok = (G == 1 && (sig[0] == 12844 || sig[0] == 12833)) || is(6444, 6433) || is(6433, 6422);
  if (!ok) return kNotHandled;
  // every staged array is read by bulk copies, which need 16-byte aligned sources
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  for (int g = 0; g < G; ++g)
    if (!a16(kc[g].codes) || !a16(vc[g].codes) || !a16(kc[g].norm) || !a16(kc[g].rnorm) || !a16(vc[g].norm))
      return kNotHandled;

  const DecodeWs W = decode_ws(B, Hq, Hkv, D, G, max_len);
  if (W.nsplit > kMergeMaxSplit) return kNotHandled;
  char* base = static_cast<char*>(ws);
  float* qp = reinterpret_cast<float*>(base + W.qp);
  float* part = reinterpret_cast<float*>(base + W.part);
  {   // every group of an instantiated kernel has the same width (64 or 128)
    int r = launch_prep(q, q_dtype, B * Hq, kctx, off, G, qp, D, perm, Hq, Hq / Hkv, st);
    if (r != TQ_OK) return r;
  }
  MmaArgs A{};
  A.B = B; A.Hq = Hq; A.Hkv = Hkv; A.D = D; A.nsplit = W.nsplit; A.chunk = W.chunk; A.G = G;
  A.rep = Hq / Hkv;
  A.nsub = (A.rep + kRep - 1) / kRep;
  A.max_len = max_len; A.scale_log2 = scale * 1.4426950408889634f; A.seq_lens = seq_lens;
  A.qprep = qp; A.part = part; A.part_ld = W.part_ld;
  for (int g = 0; g < G; ++g) {
    MmaGroup& gr = A.g[g];
    gr.kcodes = kc[g].codes; gr.knorm = kc[g].norm; gr.krnorm = kc[g].rnorm;
    gr.vcodes = vc[g].codes; gr.vnorm = vc[g].norm;
    gr.kc_inv = host_luts(kctx[g], vctx[g], &gr.lut);
    gr.coef = kctx[g]->sqrt_pi_over_2_over_m;
    gr.off = off[g];
    gr.kcap = kc[g].cap;
    gr.vcap = vc[g].cap;
  }
  A.err = kctx[0]->dev_err;
  A.table = table;
  if (table) {
    A.page = page;
    A.max_pages = (int)(max_len / page);
    int64_t pool = INT64_MAX;
    for (int g = 0; g < G; ++g) pool = std::min(pool, std::min(kc[g].cap, vc[g].cap));
    A.npages = pool / ((int64_t)Hkv * page);
  }
  for (int g = 0; g < G; ++g) {
    A.piv[g] = vctx[g]->Pi;
    A.piv_bytes[g] = (uint32_t)(vctx[g]->lay.d * vctx[g]->lay.d * sizeof(float));
  }
  int r;
  if (G == 1 && sig[0] == 12844) r = launch_mma_t<C128_44, void>(A, W.nsplit, B * Hkv * A.nsub, st);
  else if (G == 1) r = launch_mma_t<C128_33, void>(A, W.nsplit, B * Hkv * A.nsub, st);
  else if (is(6444, 6433)) r = launch_mma_t<C64_44, C64_33>(A, W.nsplit, B * Hkv * A.nsub, st);
  else r = launch_mma_t<C64_33, C64_22>(A, W.nsplit, B * Hkv * A.nsub, st);
  if (r != TQ_OK) return r;
  Merge2Args M{};
  M.part = part; M.part_ld = W.part_ld; M.nsplit = W.nsplit; M.D = D; M.G = G; M.out = out; M.err = A.err;
  M.perm = perm; M.Hq = Hq; M.rep = Hq / Hkv;
  for (int g = 0; g < G; ++g) { M.off[g] = off[g]; M.PiV[g] = vctx[g]->Pi; }
  M.off[G] = D;
  M.Hkv = Hkv;
  M.nsub = A.nsub;
  int pi_floats = 0;
  for (int g = 0; g < G; ++g) pi_floats += (M.off[g + 1] - M.off[g]) * (M.off[g + 1] - M.off[g]);
  M.pi_floats = pi_floats;
  const int64_t parts_bytes = (int64_t)kRep * W.part_ld * (int64_t)sizeof(float);
  M.stage_parts = parts_bytes <= 128 * 1024 ? 1 : 0;
  const int mdyn = pi_floats * (int)sizeof(float) + (M.stage_parts ? (int)parts_bytes : 0);
  cudaError_t em = ensure_smem_attrs<decode_merge_heads_kernel>(mdyn, true);
  if (em != cudaSuccess) return cuda_fail(em, "cudaFuncSetAttribute(decode_merge_heads_kernel)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * Hkv * A.nsub);
  cfg.blockDim = dim3(kMergeHThreads);
  cfg.dynamicSmemBytes = mdyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_merge_heads_kernel, M);
  count_launch();
  if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(decode_merge_heads_kernel)");
  return check_launch("decode_merge_heads_kernel");
}

// Standalone logits for prod contexts with d in {64, 128} and 2..4 code bits: workspace
// holds the prepared queries in fp32 ([nq][2d]); kNotHandled otherwise.
size_t logits_mma_workspace(int64_t nq, int d) { return (size_t)nq * 2 * d * sizeof(float); }

int launch_logits_mma(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* keys, int64_t n, float* out,
                      void* ws, cudaStream_t st) {
  const int d = ctx->lay.d, P = ctx->lay.planes;
  if (ctx->mode != TQ_MODE_PROD || (d != 64 && d != 128) || P < 2 || P > 4) return kNotHandled;
  if (nq > (int64_t)kRep * 65535) return kNotHandled;
  if ((reinterpret_cast<uintptr_t>(keys->codes) & 15) != 0) return kNotHandled;
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0)   // the prepared queries are read 16 bytes at a time
    return fail(TQ_ERR_INVALID_ARG, "attn_logits: the workspace must be 16-byte aligned");
  float* qprep = static_cast<float*>(ws);
  int r = launch_prepare_queries(ctx, q, TQ_DTYPE_F32, nq, d, qprep, 2 * d, st);
  if (r != TQ_OK) return r;
  LogitArgs A{};
  A.codes = keys->codes; A.norm = keys->norm; A.rnorm = keys->rnorm; A.qprep = qprep;
  A.n = n; A.nq = (int)nq; A.d = d; A.coef = ctx->sqrt_pi_over_2_over_m; A.out = out;
  const Codebook& cb = ctx->cb;
  for (int code = 0; code < cb.K && code < 8; ++code) {
    const __half h = __float2half_rn(cb.cc[code]);
    const __half lo = __float2half_rn(cb.cc[code] - __half2float(h));
    const uint16_t bh = *reinterpret_cast<const uint16_t*>(&h), bl = *reinterpret_cast<const uint16_t*>(&lo);
    A.ch[0][code / 4] |= (uint32_t)(bh & 0xFF) << (8 * (code % 4));
    A.ch[1][code / 4] |= (uint32_t)(bh >> 8) << (8 * (code % 4));
    A.cl[0][code / 4] |= (uint32_t)(bl & 0xFF) << (8 * (code % 4));
    A.cl[1][code / 4] |= (uint32_t)(bl >> 8) << (8 * (code % 4));
  }
  if (d == 128 && P == 4) return launch_logits_t<GroupCfg<128, 4, 4>>(A, st);
  if (d == 128 && P == 3) return launch_logits_t<GroupCfg<128, 3, 3>>(A, st);
  if (d == 128) return launch_logits_t<GroupCfg<128, 2, 2>>(A, st);
  if (P == 4) return launch_logits_t<GroupCfg<64, 4, 4>>(A, st);
  if (P == 3) return launch_logits_t<GroupCfg<64, 3, 3>>(A, st);
  return launch_logits_t<GroupCfg<64, 2, 2>>(A, st);
}

}  // namespace tq
