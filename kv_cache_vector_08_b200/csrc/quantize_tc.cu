// Quantize on the 5th-generation tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// turboquant.net "Quant / DeQuant 函数": y = Pi x, nearest Lloyd-Max centroid per rotated
// coordinate; admirer.cn QJL paragraph: signs of the projected residual.  For a tile of
// 128 vectors the two projections are dense contractions:
//
//   D_y [128 x d] = X [128 x d] * Pi^T            x bf16 (exact), Pi = Pi_hi + Pi_mid + Pi_lo (bf16)
//   D_z [128 x d] = R [128 x d] * M^T             R = r * 2^8 (fp16 hi + lo), M * 2^4 (fp16 hi + lo)
//
// Pi x is fp32-accurate (three bf16 splits of Pi against the exact bf16 input), so the
// norm comes for free as ||Pi x|| = ||x||.  The residual r = y - c[idx] lives in the
// rotated basis, and S r = (S Pi^T) y-residual = M r, so the QJL projection is a second
// GEMM with A taken straight from tensor memory (hi*hi + hi*lo + lo*hi products).
//
// Roles (576 threads, one persistent CTA per SM): warp 0 issues TMA loads (constants
// once, then the x tiles one 128-byte K atom at a time), warp 1 allocates TMEM and issues
// the MMAs, warps 2-17 are the epilogue: thread (row, w) owns vector `row` of the tile and
// coordinates [w d/4, (w+1) d/4), i.e. exactly one quarter of its packed record.  Two TMEM
// accumulator buffers (each holding a tile's Pi x, then its QJL projection) and two
// residual buffers let the MMAs of the next tile run under the epilogue of this one.
// Every mbarrier wait is bounded; a timeout sets the context's error word and the CTA
// winds down (in-flight copies and MMAs are drained and TMEM is always released).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr uint64_t kWaitNs = 2000000000ull;   // a pipeline wait longer than 2 s is declared stuck
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColBuf0 = 0, kColR0 = 256;  // accumulators [2] x 128 cols, residuals [2] x 128 cols
constexpr float kRScale = 256.f;              // the residual enters the QJL GEMM as r * 2^8 (M as 16 * M)
constexpr int kEpiWarps = 16;                 // 4 warpgroups: thread = (vector row, quarter of its coords)
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;

struct QtArgs {
  int64_t n;
  const int64_t* slots;
  uint8_t* codes;
  uint16_t* norm;
  uint16_t* rnorm;
  int* err;
  // symmetric codebook: boundaries t[L/2-1+j] = pos_t[j-1] (j >= 1, the middle one is 0),
  // centroids c[L/2+j] = mag[j] = -c[L/2-1-j]
  float pos_t[8];
  float mag[8];
};

// Shared-memory plan (operand regions 1024-byte aligned); x is staged per 128-byte K atom
// (128 rows x 64 columns bf16 = 16 KB) so loads of the next tile overlap the MMAs.
template <int D, bool PROD>
struct Smem {
  static constexpr int KA = D / 64;
  static constexpr int ATOM = kTileM * 128;
  static constexpr int PI_SPLIT = D * D * 2;
  static constexpr int M_SPLIT = D * D * 2;
  static constexpr int NSLOT = (D == 128 && PROD) ? 3 : 4;
  static constexpr int OFF_PI = 0;
  static constexpr int OFF_M = OFF_PI + 3 * PI_SPLIT;
  static constexpr int OFF_X = OFF_M + (PROD ? 2 * M_SPLIT : 0);
  static constexpr int OFF_XCH = OFF_X + NSLOT * ATOM;          // float [2][4][128] x 2 (norm partials)
  static constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 4 * kTileM * 4;
  static constexpr int BYTES = OFF_BAR + 256 + 1024;            // barriers + alignment slack
};

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D, bool PROD, int K>
__global__ void __launch_bounds__(kThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_pi,
                                                                  const __grid_constant__ CUtensorMap tm_m, QtArgs A) {
  using SM = Smem<D, PROD>;
  constexpr int KA = SM::KA, NSLOT = SM::NSLOT;
  constexpr int NK = D / 16;             // k-steps per product
  constexpr int CQ = D / 4;              // coordinates per epilogue thread (one record quarter)
  constexpr int LEVELS = 1 << K;
  constexpr int P = K + (PROD ? 1 : 0);  // bit planes
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_n = reinterpret_cast<float*>(smem + SM::OFF_XCH);          // [2][4][128] partial ||y||^2
  float* s_rn = s_n + 2 * 4 * kTileM;                                  // [2][4][128] partial ||r||^2
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);
  uint64_t* full_x = bars;                  // [NSLOT] TMA -> MMA
  uint64_t* empty_x = bars + NSLOT;         // [NSLOT] MMA -> TMA
  uint64_t* const_full = bars + 2 * NSLOT;  // constant operands landed
  // Every barrier below exists once per accumulator buffer: a barrier completes its next
  // phase only after each of its waiters has seen the previous one, so parity waits never
  // skip a phase even when one role runs a whole tile ahead of another.
  uint64_t* y_full = const_full + 1;        // [2] MMA -> epilogue (Pi x ready)
  uint64_t* z_full = y_full + 2;            // [2] MMA -> epilogue (QJL projection ready)
  uint64_t* r_full = z_full + 2;            // [2] epilogue -> MMA (residual in TMEM)
  uint64_t* buf_empty = r_full + 2;         // [2] epilogue -> MMA (accumulator buffer free)
  uint64_t* xn = buf_empty + 2;             // [2] norm partials written
  uint64_t* xr = xn + 2;                    // [2] residual-norm partials written
  uint64_t* drain = xr + 2;                 // MMA issuer: every issued MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (A.n + kTileM - 1) / kTileM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(full_x + s, 1);
      mbar_init(empty_x + s, 1);
    }
    mbar_init(const_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(y_full + b, 1);
      mbar_init(z_full + b, 1);
      mbar_init(r_full + b, kEpiThreads);
      mbar_init(buf_empty + b, kEpiThreads);
      mbar_init(xn + b, kEpiThreads);
      mbar_init(xr + b, kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const volatile int* abort_v = abort_flag;
  auto fail = [&](int code) {
    atomicExch(abort_flag, 1);
    if (A.err) atomicCAS(A.err, 0, code);
  };
  auto wait = [&](uint64_t* bar, uint32_t parity) { return mbar_wait(bar, parity, abort_v, kWaitNs); };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      mbar_arrive_expect_tx(const_full, 3 * SM::PI_SPLIT + (PROD ? 2 * SM::M_SPLIT : 0));
      for (int s = 0; s < 3; ++s)
        for (int a = 0; a < KA; ++a)
          tma_load_2d(smem + SM::OFF_PI + s * SM::PI_SPLIT + a * D * 128, &tm_pi, 64 * a, s * D, const_full);
      if (PROD)
        for (int s = 0; s < 2; ++s)
          for (int a = 0; a < KA; ++a)
            tma_load_2d(smem + SM::OFF_M + s * SM::M_SPLIT + a * D * 128, &tm_m, 64 * a, s * D, const_full);
      int pending[NSLOT];                 // parity of the load in flight in each slot, -1: none
      for (int s = 0; s < NSLOT; ++s) pending[s] = -1;
      int64_t q = 0;                      // atom loads issued
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        for (int a = 0; a < KA; ++a, ++q) {
          const int s = (int)(q % NSLOT);
          const uint32_t ph = (uint32_t)((q / NSLOT) & 1);
          if (!wait(empty_x + s, ph ^ 1)) { fail(101); ok = false; break; }
          mbar_arrive_expect_tx(full_x + s, SM::ATOM);
          tma_load_2d(smem + SM::OFF_X + s * SM::ATOM, &tm_x, 64 * a, (int)(tile * kTileM), full_x + s);
          pending[s] = (int)ph;
        }
      }
      // copies still in flight land before the CTA releases its shared memory
      mbar_wait(const_full, 0, nullptr, kWaitNs);
      for (int s = 0; s < NSLOT; ++s)
        if (pending[s] >= 0) mbar_wait(full_x + s, (uint32_t)pending[s], nullptr, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idy = idesc_f16(kTileM, D, 1), idz = idesc_f16(kTileM, D, 0);
      const uint32_t pi_addr = smem_u32(smem + SM::OFF_PI), m_addr = smem_u32(smem + SM::OFF_M);
      bool ok = wait(const_full, 0);
      if (!ok) fail(102);
      // z = (R_hi + R_lo)(M_hi + M_lo) without the lo*lo term, into the tile's buffer
      auto issue_z = [&](int t) -> bool {
        const int par = t & 1;
        if (!wait(r_full + par, (uint32_t)((t >> 1) & 1))) { fail(104); return false; }
        tc_fence_after();
        const uint32_t dz = tmem + kColBuf0 + 128 * par, rz = tmem + kColR0 + 128 * par;
        for (int sp = 0; sp < 3; ++sp) {
          const uint32_t a_col = rz + (sp == 2 ? D / 2 : 0);
          const int msp = (sp == 1) ? 1 : 0;
          for (int ks = 0; ks < NK; ++ks) {
            const uint64_t db = desc_sw128(m_addr + msp * SM::M_SPLIT + (ks >> 2) * D * 128 + (ks & 3) * 32);
            mma_ts(dz, a_col + ks * 8, db, idz, (sp | ks) ? 1u : 0u);
          }
        }
        mma_commit(z_full + par);
        return true;
      };
      int it = 0;
      int64_t q = 0;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++it) {
        const int par = it & 1;
        if (!wait(buf_empty + par, (uint32_t)(((it >> 1) & 1) ^ 1))) { fail(103); ok = false; break; }
        tc_fence_after();
        const uint32_t dy = tmem + kColBuf0 + 128 * par;
        for (int a = 0; a < KA; ++a, ++q) {
          const int s = (int)(q % NSLOT);
          if (!wait(full_x + s, (uint32_t)((q / NSLOT) & 1))) { fail(103); ok = false; break; }
          tc_fence_after();
          const uint32_t x_addr = smem_u32(smem + SM::OFF_X + s * SM::ATOM);
          for (int sp = 0; sp < 3; ++sp)
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t da = desc_sw128(x_addr + kk * 32);
              const uint64_t db = desc_sw128(pi_addr + sp * SM::PI_SPLIT + a * D * 128 + kk * 32);
              mma_ss(dy, da, db, idy, (a | sp | kk) ? 1u : 0u);
            }
          mma_commit(empty_x + s);
        }
        if (!ok) break;
        mma_commit(y_full + par);
        if (PROD && it >= 1 && !issue_z(it - 1)) { ok = false; break; }
      }
      if (PROD && ok && it >= 1) issue_z(it - 1);
      // every MMA issued above completes before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------------------ epilogue
    const int ew = warp - 2, wg = ew >> 2;             // wg: which quarter of the coordinates
    const int tq = warp & 3;                           // TMEM lanes 32*tq .. +31
    const int row = tq * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(tq * 32) << 16);
    const int c0 = wg * CQ;
    // state of the tile whose QJL signs are still to come
    uint32_t pend_planes[K];
    float pend_n = 0.f;
    int64_t pend_v = -1;
    auto load_cols = [&](uint32_t col, float (&v)[CQ]) {
      if constexpr (CQ == 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + col, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      } else {
        uint32_t r[16];
        tmem_ld16(lane_base + col, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
      }
    };
    // one record quarter: planes[0..P-1] of this thread's CQ coordinates
    auto store_quarter = [&](int64_t v, const uint32_t* pl, float nrm, float rn2) {
      if (v >= A.n) return;
      const int64_t slot = A.slots ? A.slots[v] : v;
      uint8_t* rec = A.codes + slot * (int64_t)(P * D / 8) + wg * (P * D / 32);
      if constexpr (CQ == 32) {
        if constexpr (P == 4) *reinterpret_cast<uint4*>(rec) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
        else if constexpr (P == 2) *reinterpret_cast<uint2*>(rec) = make_uint2(pl[0], pl[1]);
        else
#pragma unroll
          for (int p = 0; p < P; ++p) reinterpret_cast<uint32_t*>(rec)[p] = pl[p];
      } else {
        if constexpr (P == 4) *reinterpret_cast<uint2*>(rec) = make_uint2(pl[0] | (pl[1] << 16), pl[2] | (pl[3] << 16));
        else if constexpr (P == 2) *reinterpret_cast<uint32_t*>(rec) = pl[0] | (pl[1] << 16);
        else
#pragma unroll
          for (int p = 0; p < P; ++p) reinterpret_cast<uint16_t*>(rec)[p] = (uint16_t)pl[p];
      }
      if (wg == 0) {
        A.norm[slot] = __half_as_ushort(__float2half_rn(nrm));
        if (PROD) A.rnorm[slot] = nrm > 0.f ? __half_as_ushort(__float2half_rn(sqrtf(rn2))) : (uint16_t)0;
      }
    };
    // signs of tile t's QJL projection, then its record quarter
    auto finish_z = [&](int t) -> bool {
      const int par = t & 1;
      if (!wait(z_full + par, (uint32_t)((t >> 1) & 1))) { fail(106); return false; }
      tc_fence_after();
      float z[CQ];
      load_cols(kColBuf0 + 128 * par + c0, z);
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < CQ; ++i) w |= (z[i] >= 0.f ? 1u : 0u) << i;
      if (pend_n == 0.f) w = (CQ == 32) ? 0xFFFFFFFFu : 0xFFFFu;   // zero vector: all signs +1
      float rn2 = 0.f;
      if (wg == 0) {
        if (!wait(xr + par, (uint32_t)((t >> 1) & 1))) { fail(107); return false; }
#pragma unroll
        for (int g = 0; g < 4; ++g) rn2 += s_rn[(par * 4 + g) * kTileM + row];
      }
      tc_fence_before();
      mbar_arrive(buf_empty + par);
      uint32_t pl[P];
#pragma unroll
      for (int p = 0; p < K; ++p) pl[p] = pend_planes[p];
      pl[P - 1] = w;
      store_quarter(pend_v, pl, pend_n, rn2);
      return true;
    };
    int it = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const int par = it & 1;
      if (!wait(y_full + par, (uint32_t)((it >> 1) & 1))) { fail(105); ok = false; break; }
      tc_fence_after();
      float y[CQ];
      load_cols(kColBuf0 + 128 * par + c0, y);
      float n2p = 0.f;
#pragma unroll
      for (int i = 0; i < CQ; ++i) n2p = fmaf(y[i], y[i], n2p);
      s_n[(par * 4 + wg) * kTileM + row] = n2p;
      mbar_arrive(xn + par);
      if (!wait(xn + par, (uint32_t)((it >> 1) & 1))) { fail(108); ok = false; break; }
      float n2 = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) n2 += s_n[(par * 4 + g) * kTileM + row];
      const float nrm = sqrtf(n2);
      // nearest centroid by sign and magnitude: y = D / ||x|| > 0 picks the upper half of the
      // (odd-symmetric) codebook; the magnitude index is a binary search of |D| against the
      // positive boundaries scaled by ||x|| (so no division per coordinate)
      float pn[8];
#pragma unroll
      for (int j = 0; j < LEVELS / 2 - 1; ++j) pn[j] = nrm * A.pos_t[j];
      const float s256 = nrm > 0.f ? kRScale / nrm : 0.f;   // residual scale r * 2^8 = D s256 - 2^8 c
      uint32_t S = 0u, B0 = 0u, B1 = 0u, B2 = 0u;
      float rn2p = 0.f;
      float rs[CQ];
#pragma unroll
      for (int i = 0; i < CQ; ++i) {
        const float Dv = y[i], a = fabsf(Dv);
        const bool sp = Dv > 0.f;
        bool b0 = false, b1 = false, b2 = false;
        float m = 0.f;
        if constexpr (K == 1) {
          if (PROD) m = A.mag[0];
        } else if constexpr (K == 2) {
          b0 = a > pn[0];
          if (PROD) m = b0 ? A.mag[1] : A.mag[0];
        } else if constexpr (K == 3) {
          b1 = a > pn[1];
          b0 = a > (b1 ? pn[2] : pn[0]);
          if (PROD) m = b1 ? (b0 ? A.mag[3] : A.mag[2]) : (b0 ? A.mag[1] : A.mag[0]);
        } else {
          b2 = a > pn[3];
          b1 = a > (b2 ? pn[5] : pn[1]);
          b0 = a > (b2 ? (b1 ? pn[6] : pn[4]) : (b1 ? pn[2] : pn[0]));
          if (PROD)
            m = b2 ? (b1 ? (b0 ? A.mag[7] : A.mag[6]) : (b0 ? A.mag[5] : A.mag[4]))
                   : (b1 ? (b0 ? A.mag[3] : A.mag[2]) : (b0 ? A.mag[1] : A.mag[0]));
        }
        S |= (uint32_t)sp << i;
        B0 |= (uint32_t)b0 << i;
        B1 |= (uint32_t)b1 << i;
        B2 |= (uint32_t)b2 << i;
        if (PROD) {
          const float r = fmaf(Dv, s256, sp ? -kRScale * m : kRScale * m);   // 2^8 (y - c[idx])
          rn2p = fmaf(r, r, rn2p);
          rs[i] = r;
        }
      }
      rn2p *= 1.f / (kRScale * kRScale);
      // idx = L/2 + |idx| (y > 0) or L/2 - 1 - |idx| = (L/2 - 1) ^ |idx| (y <= 0):
      // bit K-1 is the sign, the lower bits are the magnitude bits, flipped when y <= 0
      uint32_t planes[P];
      {
        const uint32_t nS = ~S;
        if constexpr (K >= 2) planes[0] = B0 ^ nS;
        if constexpr (K >= 3) planes[1] = B1 ^ nS;
        if constexpr (K >= 4) planes[2] = B2 ^ nS;
        planes[K - 1] = S;
        if constexpr (CQ == 16) {
#pragma unroll
          for (int p = 0; p < K; ++p) planes[p] &= 0xFFFFu;
        }
      }
      const int64_t v = tile * kTileM + row;
      if (PROD) {
        uint32_t hi[CQ / 2], lo[CQ / 2];
#pragma unroll
        for (int i = 0; i < CQ / 2; ++i) {
          const float a0 = rs[2 * i], a1 = rs[2 * i + 1];
          const float h0 = __half2float(__float2half_rn(a0)), h1 = __half2float(__float2half_rn(a1));
          hi[i] = pack_h2(h0, h1);
          lo[i] = pack_h2(a0 - h0, a1 - h1);
        }
        const uint32_t rz = lane_base + kColR0 + 128 * par + c0 / 2;
        if constexpr (CQ == 32) {
          tmem_st16(rz, hi);
          tmem_st16(rz + D / 2, lo);
        } else {
          tmem_st8(rz, hi);
          tmem_st8(rz + D / 2, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(r_full + par);
        s_rn[(par * 4 + wg) * kTileM + row] = rn2p;
        mbar_arrive(xr + par);
        if (it >= 1 && !finish_z(it - 1)) { ok = false; break; }
#pragma unroll
        for (int p = 0; p < K; ++p) pend_planes[p] = planes[p];
        pend_n = nrm;
        pend_v = v;
      } else {
        tc_fence_before();
        mbar_arrive(buf_empty + par);
        store_quarter(v, planes, nrm, 0.f);
      }
    }
    if (PROD && ok && it >= 1) finish_z(it - 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// 2-D row-major map [rows][cols] of 16-bit elements, box {64 columns, box_rows rows},
// 128-byte swizzle (the canonical K-major operand layout of tcgen05.mma).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
              uint64_t row_stride_bytes, uint32_t box_rows) {
  EncodeTiled enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool PROD, int K>
int launch_tc_t(const tq_ctx* ctx, const void* x, int64_t n, int64_t ld, const tq_packed* dst, const int64_t* slots,
                cudaStream_t st) {
  using SM = Smem<D, PROD>;
  CUtensorMap tx, tp, tm;
  if (!make_map(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)n, D, (uint64_t)ld * 2, kTileM))
    return fail(TQ_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled rejected the input (needs 16-byte aligned rows)");
  if (!make_map(&tp, ctx->Pi_split, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3 * D, D, D * 2, D))
    return fail(TQ_ERR_INTERNAL, "tensor map for Pi splits");
  if (PROD) {
    if (!make_map(&tm, ctx->M_split, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * D, D, D * 2, D))
      return fail(TQ_ERR_INTERNAL, "tensor map for M splits");
  } else {
    tm = tp;
  }
  QtArgs a{};
  a.n = n;
  a.slots = slots;
  a.codes = dst->codes;
  a.norm = dst->norm;
  a.rnorm = dst->rnorm;
  a.err = ctx->dev_err;
  const int L = ctx->cb.K;
  for (int j = 0; j < 8; ++j) {
    a.pos_t[j] = (j + 1 < L / 2) ? ctx->cb.t[L / 2 - 1 + j + 1] : INFINITY;
    a.mag[j] = (j < L / 2) ? ctx->cb.c[L / 2 + j] : 0.f;
  }
  auto kern = quantize_tc_kernel<D, PROD, K>;
  // one CTA per SM: it owns all 512 TMEM columns (more than half the shared memory forces it)
  const int smem_bytes = SM::BYTES > 120 * 1024 ? SM::BYTES : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(quantize_tc)");
  const int64_t ntiles = (n + kTileM - 1) / kTileM;
  int sms = 148;
  int dev = ctx->device;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::min<int64_t>(ntiles, sms);
  kern<<<grid, kThreads, smem_bytes, st>>>(tx, tp, tm, a);
  count_launch();
  return check_launch("quantize_tc_kernel");
}

}  // namespace

// bf16 input, d in {64, 128}, k in [1, 4]; other shapes return kNotHandled.
int launch_quantize_tc(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                       const int64_t* slots, cudaStream_t st) {
  if (x_dtype != TQ_DTYPE_BF16 || !ctx->Pi_split) return kNotHandled;
  const int d = ctx->lay.d, k = ctx->lay.k;
  if ((d != 64 && d != 128) || (ld * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(x) % 16) != 0) return kNotHandled;
  if (n < kTileM) return kNotHandled;   // small batches: the CUDA-core kernel
  const bool prod = ctx->mode == TQ_MODE_PROD;
#define TQ_TC_CASE(DD, PP, KK) \
  if (d == DD && prod == PP && k == KK) return launch_tc_t<DD, PP, KK>(ctx, x, n, ld, dst, slots, st);
  TQ_TC_CASE(128, true, 3) TQ_TC_CASE(128, true, 2) TQ_TC_CASE(128, true, 1)
  TQ_TC_CASE(128, false, 4) TQ_TC_CASE(128, false, 3) TQ_TC_CASE(128, false, 2)
  TQ_TC_CASE(64, true, 3) TQ_TC_CASE(64, true, 2) TQ_TC_CASE(64, true, 1)
  TQ_TC_CASE(64, false, 4) TQ_TC_CASE(64, false, 3) TQ_TC_CASE(64, false, 2)
#undef TQ_TC_CASE
  return kNotHandled;
}

}  // namespace tq
