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
// Roles (608 threads, one persistent CTA per SM): warp 0 issues TMA loads (constants
// once, then the x tiles one 128-byte K atom at a time), warp 1 allocates TMEM and issues
// the Pi x MMAs, warp 18 issues the QJL MMAs (so they wait only for their residual, never
// for the next x tile), warps 2-17 are the epilogue: thread (row, w) owns vector `row` of the tile and
// coordinates [w d/4, (w+1) d/4), i.e. exactly one quarter of its packed record.  TMEM
// holds two Pi x accumulators (each released as soon as the epilogue has read it, so the
// Pi x GEMM runs two tiles ahead), one QJL accumulator and one residual operand: the QJL
// GEMM of tile t runs under the epilogue of tile t + 1, which collects its signs.
// Every mbarrier wait is bounded; a timeout sets the context's error word and the CTA
// winds down (in-flight copies and MMAs are drained and TMEM is always released).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace tq {

// ------------------------------------------------------------------- tensor maps (host)
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

// 2-D row-major map [rows][cols] of dt elements, box {box_cols, box_rows}, no swizzle.
bool make_map_plain(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiled enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
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

namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr uint64_t kWaitNs = 2000000000ull;   // a pipeline wait longer than 2 s is declared stuck
constexpr uint32_t kTmemCols = 512;   // columns [0, 2d): Pi x [2]; [2d, 3d): QJL projection; [3d, 4d): residual
constexpr float kRScale = 256.f;              // the residual enters the QJL GEMM as r * 2^8 (M as 16 * M)
constexpr int kEpiWarps = 16;                 // 4 warpgroups: thread = (vector row, quarter of its coords)
constexpr int kThreads = 96 + 32 * kEpiWarps;   // + TMA warp, Pi x issuer warp, QJL issuer warp (last)
constexpr int kZWarp = 2 + kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;

struct QtArgs {
  int64_t n;
  int64_t cap;            // slots in the packed storage (a slot outside [0, cap) is skipped)
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
  static constexpr int OFF_PI = 0;
  static constexpr int OFF_M = OFF_PI + 3 * PI_SPLIT;
  static constexpr int OFF_X = OFF_M + (PROD ? 2 * M_SPLIT : 0);
  // as many x slots as the 227 KB of shared memory leave (the loads take microseconds, so
  // every extra slot is prefetch depth), at most 8
  // d = 64: code words shared by the two threads of a 32-coordinate group meet here
  static constexpr int XW = D == 64 ? 2 * kTileM * 4 * 3 * 4 : 0;   // uint32 [2][128][4][3]
  static constexpr int FIXED = OFF_X + 2 * 2 * 4 * kTileM * 4 + XW + 512 + 1024;
  static constexpr int NSLOT = (232448 - FIXED) / ATOM > 8 ? 8 : (232448 - FIXED) / ATOM;
  static constexpr int OFF_XCH = OFF_X + NSLOT * ATOM;          // float [2][4][128] x 2 (norm partials)
  static constexpr int OFF_XW = OFF_XCH + 2 * 2 * 4 * kTileM * 4;
  static constexpr int OFF_BAR = OFF_XW + XW;
  static constexpr int BYTES = OFF_BAR + 512 + 1024;            // barriers + alignment slack
};

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The epilogue's comparisons and bit packing run on the FMA pipe (the integer / compare
// pipe has half its issue rate): with B = 2^64, sat(|y| B - t B) is exactly [|y| > t]
// (every nonzero difference of floats near t is far above 2^-64), a selected threshold is
// an FMA of 0/1 values, and packed bits accumulate exactly as sums of powers of two in
// 16-bit halves of each word.
constexpr float kBig = 18446744073709551616.f;   // 2^64

__device__ __forceinline__ float above(float y, float nt) {   // [|y| > t], nt = -t 2^64
  float d;
  asm("{\n .reg .f32 a;\n abs.f32 a, %1;\n fma.rn.sat.f32 %0, a, %2, %3;\n}\n" : "=f"(d) : "f"(y), "f"(kBig), "f"(nt));
  return d;
}
// [y > 0] for every normal y; a denormal y (within 2^-126 of the sign boundary) counts as 0
__device__ __forceinline__ float positive(float y) {
  float d;
  asm("mul.rn.ftz.sat.f32 %0, %1, %2;\n" : "=f"(d) : "f"(y), "f"(8.5070591730234616e37f));   // 2^126
  return d;
}

// Two fp32 lanes in one 64-bit register (Blackwell's packed f32x2 FMA: one issue slot
// for two coordinates).
using f2 = unsigned long long;
__device__ __forceinline__ f2 f2pack(float a, float b) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2split(f2 r, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;\n" : "=f"(a), "=f"(b) : "l"(r)); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 bcast2(float a) { return f2pack(a, a); }

// Bit-packing accumulators: half-words of PW words as exact float sums.
template <int PW>
struct PackAcc {
  float h[2 * PW];
  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int i = 0; i < 2 * PW; ++i) h[i] = 0.f;
  }
  // start from the bits in `mask` set (they are cleared with sub())
  __device__ __forceinline__ void set(const uint32_t (&mask)[PW]) {
#pragma unroll
    for (int i = 0; i < PW; ++i) {
      h[2 * i] = (float)(mask[i] & 0xFFFFu);
      h[2 * i + 1] = (float)(mask[i] >> 16);
    }
  }
  __device__ __forceinline__ void sub(int q, float v) { h[q >> 4] = fmaf(v, -(float)(1u << (q & 15)), h[q >> 4]); }
  // add v (0 or 1) at bit q = 32 word + bit
  __device__ __forceinline__ void add(int q, float v) { h[q >> 4] = fmaf(v, (float)(1u << (q & 15)), h[q >> 4]); }
  __device__ __forceinline__ void to_words(uint32_t (&w)[PW]) const {
#pragma unroll
    for (int i = 0; i < PW; ++i) {
      const uint32_t lo = __float_as_uint(h[2 * i] + 8388608.f), hi = __float_as_uint(h[2 * i + 1] + 8388608.f);
      w[i] = __byte_perm(lo, hi, 0x5410);
    }
  }
};

template <int D, bool PROD, int K>
__global__ void __launch_bounds__(kThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_pi,
                                                                  const __grid_constant__ CUtensorMap tm_m, QtArgs A) {
  using SM = Smem<D, PROD>;
  constexpr int KA = SM::KA, NSLOT = SM::NSLOT;
  constexpr int NK = D / 16;             // k-steps per product
  constexpr int CQ = D / 4;              // coordinates per epilogue thread (one record quarter)
  constexpr int LEVELS = 1 << K;
  constexpr int P = K + (PROD ? 1 : 0);  // code bits per coordinate
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_n = reinterpret_cast<float*>(smem + SM::OFF_XCH);          // [2][4][128] partial ||y||^2
  float* s_rn = s_n + 2 * 4 * kTileM;                                  // [2][4][128] partial ||r||^2
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);
  uint64_t* full_x = bars;                  // [NSLOT] TMA -> MMA
  uint64_t* empty_x = bars + NSLOT;         // [NSLOT] MMA -> TMA
  uint64_t* const_full = bars + 2 * NSLOT;  // constant operands landed
  // A barrier completes its next phase only after each of its waiters has seen the
  // previous one (every chain below closes through the other role), so parity waits never
  // skip a phase even when one role runs ahead of another.
  uint64_t* y_full = const_full + 1;        // [2] MMA -> epilogue (Pi x ready)
  uint64_t* y_empty = y_full + 2;           // [2] epilogue -> MMA (Pi x read into registers)
  uint64_t* z_full = y_empty + 2;           // MMA -> epilogue (QJL projection ready, residual consumed)
  uint64_t* z_empty = z_full + 1;           // epilogue -> MMA (QJL projection read)
  uint64_t* r_full = z_empty + 1;           // epilogue -> MMA (residual in TMEM)
  uint64_t* xn = r_full + 1;                // [2] norm partials written
  uint64_t* xr = xn + 2;                    // [2] residual-norm partials written
  uint64_t* drain = xr + 2;                 // [2] MMA issuers (Pi x, QJL): every issued MMA complete
  uint64_t* pairb = drain + 2;              // [8 pairs][2] d = 64: the two threads of a group met
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pairb + 16);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (A.n + kTileM - 1) / kTileM;
  // this CTA's tiles: blockIdx.x + t * gridDim.x for t < nloc
  const int nloc = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  constexpr uint32_t kColZ = 2 * D, kColR = 3 * D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(full_x + s, 1);
      mbar_init(empty_x + s, 1);
    }
    mbar_init(const_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(y_full + b, 1);
      mbar_init(y_empty + b, kEpiThreads);
      mbar_init(xn + b, kEpiThreads);
      mbar_init(xr + b, kEpiThreads);
    }
    mbar_init(z_full, 1);
    mbar_init(z_empty, kEpiThreads);
    mbar_init(r_full, kEpiThreads);
    mbar_init(drain, 1);
    mbar_init(drain + 1, 1);
    for (int i = 0; i < 16; ++i) mbar_init(pairb + i, 64);
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
    // ------------------------------------------------------------------ Pi x MMA issuer
    if (lane == 0) {
      const uint32_t idy = idesc_f16(kTileM, D, 1);
      const uint32_t pi_addr = smem_u32(smem + SM::OFF_PI);
      bool ok = wait(const_full, 0);
      if (!ok) fail(102);
      // Pi x of local tile t into accumulator t & 1 (three bf16 splits of Pi); it runs
      // two tiles ahead of the epilogue
      int64_t q = 0;                      // x atoms consumed
      for (int t = 0; ok && t < nloc; ++t) {
        const int b = t & 1;
        if (!wait(y_empty + b, (uint32_t)(((t >> 1) & 1) ^ 1))) { fail(103); break; }
        tc_fence_after();
        const uint32_t dy = tmem + (uint32_t)(b * D);
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
        mma_commit(y_full + b);
      }
      // every MMA issued above completes before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kWaitNs);
    }
  } else if (warp == kZWarp) {
    // ------------------------------------------------------------------- QJL MMA issuer
    if (PROD && lane == 0) {
      const uint32_t idz = idesc_f16(kTileM, D, 0);
      const uint32_t m_addr = smem_u32(smem + SM::OFF_M);
      bool ok = wait(const_full, 0);
      if (!ok) fail(102);
      // QJL projection of tile t: (R_hi + R_lo)(M_hi + M_lo) without the lo*lo term, as
      // soon as the epilogue has written the residual and read the previous projection
      for (int t = 0; ok && t < nloc; ++t) {
        if (!wait(r_full, (uint32_t)(t & 1))) { fail(104); break; }
        if (!wait(z_empty, (uint32_t)((t & 1) ^ 1))) { fail(104); break; }
        tc_fence_after();
        const uint32_t dz = tmem + kColZ, rz = tmem + kColR;
        for (int sp = 0; sp < 3; ++sp) {
          const uint32_t a_col = rz + (sp == 2 ? D / 2 : 0);
          const int msp = (sp == 1) ? 1 : 0;
          for (int ks = 0; ks < NK; ++ks) {
            const uint64_t db = desc_sw128(m_addr + msp * SM::M_SPLIT + (ks >> 2) * D * 128 + (ks & 3) * 32);
            mma_ts(dz, a_col + ks * 8, db, idz, (sp | ks) ? 1u : 0u);
          }
        }
        mma_commit(z_full);
      }
      mma_commit(drain + 1);
      mbar_wait(drain + 1, 0, nullptr, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------------------ epilogue
    const int ew = warp - 2, wg = ew >> 2;             // wg: which quarter of the coordinates
    const int tq = warp & 3;                           // TMEM lanes 32*tq .. +31
    const int row = tq * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(tq * 32) << 16);
    const int c0 = wg * CQ;
    // this thread's words of the packed record (the code bit places of the packed format
    // depend only on the coordinate's place inside its 32-coordinate group).  At d = 64 a
    // thread holds half a group; for 4-bit codes that is two whole words, otherwise the
    // two threads of a group share every word (SHARED): each builds the group's words
    // from its own coordinates, as if they were slices 0-1, and the pair combines them.
    constexpr bool SHARED = (D == 64 && P != 4);
    constexpr int PW = SHARED ? P : P * CQ / 32;
    uint32_t* s_xw = reinterpret_cast<uint32_t*>(smem + SM::OFF_XW);
    auto put = [](uint32_t (&w)[PW], int i, int b, bool bit) {
      const int q = code_bit_pos(P, i, b);
      w[q >> 5] |= (bit ? 1u : 0u) << (q & 31);
    };
    // state of the tile whose QJL signs are still to come
    uint32_t pend_words[PW];
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
    // this thread's PW words of the record (bytes [wg P D/32, (wg+1) P D/32)); SHARED: the
    // even thread of the pair stores the group's P words.  Every thread of both warps of
    // a pair reaches the pair barrier (rows past n only skip the global stores).
    auto store_quarter = [&](int t, int64_t v, const uint32_t (&pl)[PW], float nrm, float rn2) {
      const int tpar = t & 1;
      int64_t slot = v < A.n ? (A.slots ? A.slots[v] : v) : 0;
      const bool live = v < A.n && slot >= 0 && slot < A.cap;
      if (v < A.n && !live && wg == 0 && A.err) atomicCAS(A.err, 0, (int)kErrSlotRange);
      if (!live) slot = 0;
      if constexpr (SHARED) {
        const int odd = wg & 1;
        uint32_t w[PW];
#pragma unroll
        for (int p = 0; p < PW; ++p) w[p] = pl[p];
        if (odd) {             // slices 2-3: low-bit words two places up, top bits 4 places down
#pragma unroll
          for (int p = 0; p < PW - 1; ++p) w[p] <<= 2;
          w[PW - 1] >>= 4;
        }
        uint32_t* mine = s_xw + ((tpar * kTileM + row) * 4 + wg) * 3;
#pragma unroll
        for (int p = 0; p < PW; ++p) mine[p] = w[p];
        uint64_t* pb = pairb + ((wg >> 1) * 4 + tq) * 2 + tpar;
        mbar_arrive(pb);
        if (!wait(pb, (uint32_t)((t >> 1) & 1))) {
          fail(109);
          return;
        }
        if (!odd && live) {
          const uint32_t* other = mine + 3;
          uint32_t* rec = reinterpret_cast<uint32_t*>(A.codes + slot * (int64_t)(P * D / 8)) + (wg >> 1) * P;
#pragma unroll
          for (int p = 0; p < PW; ++p) rec[p] = w[p] | other[p];
        }
      } else if (live) {
        uint8_t* rec = A.codes + slot * (int64_t)(P * D / 8) + wg * (P * D / 32);
        if constexpr (PW == 4) *reinterpret_cast<uint4*>(rec) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
        else if constexpr (PW == 2) *reinterpret_cast<uint2*>(rec) = make_uint2(pl[0], pl[1]);
        else {
#pragma unroll
          for (int p = 0; p < PW; ++p) reinterpret_cast<uint32_t*>(rec)[p] = pl[p];
        }
      }
      if (live && wg == 0) {
        A.norm[slot] = __half_as_ushort(__float2half_rn(nrm));
        if (PROD) A.rnorm[slot] = nrm > 0.f ? __half_as_ushort(__float2half_rn(sqrtf(rn2))) : (uint16_t)0;
      }
    };
    // signs of the pending tile's QJL projection (z_full already waited) into the top code
    // bits of its words; the projection buffer is handed back to the MMA issuer
    auto take_signs = [&]() {
      tc_fence_after();
      float z[CQ];
      load_cols(kColZ + c0, z);
      tc_fence_before();
      mbar_arrive(z_empty);
      PackAcc<PW> pk;
      pk.clear();
#pragma unroll
      for (int i = 0; i < CQ; ++i) pk.add(code_bit_pos(P, i, P - 1), positive(z[i]));
      uint32_t sw[PW];
      pk.to_words(sw);
      // a projection exactly 0 sits on the sign boundary (counted positive); a zero vector
      // has all signs +1
      uint32_t topmask[PW];
#pragma unroll
      for (int p = 0; p < PW; ++p) topmask[p] = 0u;
#pragma unroll
      for (int i = 0; i < CQ; ++i) put(topmask, i, P - 1, true);
      const bool zero = pend_n == 0.f;
#pragma unroll
      for (int p = 0; p < PW; ++p) pend_words[p] |= zero ? topmask[p] : sw[p];
    };
    // the pending tile t's record words, norms last
    auto finish = [&](int t) -> bool {
      float rn2 = 0.f;
      if (wg == 0) {
        const int b = t & 1;
        if (!wait(xr + b, (uint32_t)((t >> 1) & 1))) { fail(107); return false; }
#pragma unroll
        for (int g = 0; g < 4; ++g) rn2 += s_rn[(b * 4 + g) * kTileM + row];
      }
      store_quarter(t, pend_v, pend_words, pend_n, rn2);
      return true;
    };
    // per-kernel constants: scaled negative thresholds, the 2^9 magnitude table, and the
    // places of the negative-half flags (set, then cleared for positive coordinates)
    float nt[7];
#pragma unroll
    for (int j = 0; j < 7; ++j) nt[j] = (j < LEVELS / 2 - 1) ? -kRScale * kBig * A.pos_t[j] : 0.f;
    float m2[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) m2[j] = (j < LEVELS / 2) ? 2.f * kRScale * A.mag[j] : 0.f;
    const f2 c_nt0 = bcast2(nt[0]), c_nt1 = bcast2(nt[1]), c_nt2 = bcast2(nt[2]);
    const f2 c_d20 = bcast2(nt[2] - nt[0]), c_d51 = bcast2(nt[5] - nt[1]);
    const f2 c_d40 = bcast2(nt[4] - nt[0]), c_d62 = bcast2(nt[6] - nt[2]);
    const f2 c_m1 = bcast2(-1.f), c_mhalf = bcast2(-0.5f);
    const f2 c_nm0 = bcast2(-m2[0]), c_nm2 = bcast2(-m2[2]);
    const f2 c_nd10 = bcast2(m2[0] - m2[1]), c_nd32 = bcast2(m2[2] - m2[3]);
    uint32_t nflags[PW];
#pragma unroll
    for (int p = 0; p < PW; ++p) nflags[p] = 0u;
#pragma unroll
    for (int i = 0; i < CQ; ++i) put(nflags, i, K - 1, true);
    bool ok = true;
    for (int t = 0; t < nloc; ++t) {
      const int b = t & 1;
      const int64_t tile = blockIdx.x + (int64_t)t * gridDim.x;
      if (!wait(y_full + b, (uint32_t)((t >> 1) & 1))) { fail(105); ok = false; break; }
      tc_fence_after();
      float y[CQ];
      load_cols((uint32_t)(b * D) + c0, y);
      tc_fence_before();
      mbar_arrive(y_empty + b);
      float n2p;
      {
        f2 n2 = 0ull;
#pragma unroll
        for (int i = 0; i < CQ; i += 2) {
          const f2 v = f2pack(y[i], y[i + 1]);
          n2 = fma2(v, v, n2);
        }
        float a, c;
        f2split(n2, a, c);
        n2p = a + c;
      }
      s_n[(b * 4 + wg) * kTileM + row] = n2p;
      mbar_arrive(xn + b);
      if (!wait(xn + b, (uint32_t)((t >> 1) & 1))) { fail(108); ok = false; break; }
      float n2 = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g) n2 += s_n[(b * 4 + g) * kTileM + row];
      const float nrm = sqrtf(n2);
      // nearest centroid by sign and magnitude on Y = 2^8 D / ||x|| = 2^8 y: Y > 0 picks the
      // upper half of the (odd-symmetric) codebook, a binary search of |Y| over the positive
      // boundaries gives the magnitude bits (thresholds selected by FMAs of earlier bits)
      const float s256 = nrm > 0.f ? kRScale / nrm : 0.f;
      PackAcc<PW> pk;
      pk.set(nflags);
      float rs[CQ];
      f2 rn2 = 0ull;
      const f2 S2 = bcast2(s256);
#pragma unroll
      for (int i = 0; i < CQ; i += 2) {
        float Ya, Yb;
        const f2 Y2 = mul2(f2pack(y[i], y[i + 1]), S2);
        f2split(Y2, Ya, Yb);
        const float spa = positive(Ya), spb = positive(Yb);
        float b0a = 0.f, b0b = 0.f, b1a = 0.f, b1b = 0.f, b2a = 0.f, b2b = 0.f;
        if constexpr (K == 2) {
          b0a = above(Ya, nt[0]);
          b0b = above(Yb, nt[0]);
        } else if constexpr (K == 3) {
          b1a = above(Ya, nt[1]);
          b1b = above(Yb, nt[1]);
          float ta, tb;
          f2split(fma2(f2pack(b1a, b1b), c_d20, c_nt0), ta, tb);
          b0a = above(Ya, ta);
          b0b = above(Yb, tb);
        } else if constexpr (K == 4) {
          b2a = above(Ya, nt[3]);
          b2b = above(Yb, nt[3]);
          const f2 B2 = f2pack(b2a, b2b);
          float ta, tb;
          f2split(fma2(B2, c_d51, c_nt1), ta, tb);
          b1a = above(Ya, ta);
          b1b = above(Yb, tb);
          const f2 E0 = fma2(B2, c_d40, c_nt0), E1 = fma2(B2, c_d62, c_nt2);
          f2split(fma2(f2pack(b1a, b1b), fma2(E0, c_m1, E1), E0), ta, tb);
          b0a = above(Ya, ta);
          b0b = above(Yb, tb);
        }
        // sign-magnitude index code: magnitude bits, then the negative-half flag 1 - sp
        if constexpr (K >= 2) { pk.add(code_bit_pos(P, i, 0), b0a); pk.add(code_bit_pos(P, i + 1, 0), b0b); }
        if constexpr (K >= 3) { pk.add(code_bit_pos(P, i, 1), b1a); pk.add(code_bit_pos(P, i + 1, 1), b1b); }
        if constexpr (K >= 4) { pk.add(code_bit_pos(P, i, 2), b2a); pk.add(code_bit_pos(P, i + 1, 2), b2b); }
        pk.sub(code_bit_pos(P, i, K - 1), spa);
        pk.sub(code_bit_pos(P, i + 1, K - 1), spb);
        if constexpr (PROD) {
          // -M = -2^9 |c| from the magnitude bits, then r = (Y + M/2) - sp M
          f2 NM = c_nm0;
          if constexpr (K == 2) {
            NM = fma2(f2pack(b0a, b0b), c_nd10, c_nm0);
          } else if constexpr (K == 3) {
            const f2 B0 = f2pack(b0a, b0b);
            const f2 NLO = fma2(B0, c_nd10, c_nm0), NHI = fma2(B0, c_nd32, c_nm2);
            NM = fma2(f2pack(b1a, b1b), fma2(NLO, c_m1, NHI), NLO);
          }
          const f2 R = fma2(f2pack(spa, spb), NM, fma2(c_mhalf, NM, Y2));
          rn2 = fma2(R, R, rn2);
          f2split(R, rs[i], rs[i + 1]);
        }
      }
      float rn2p;
      {
        float a, c;
        f2split(rn2, a, c);
        rn2p = a + c;
      }
      uint32_t words[PW];
      pk.to_words(words);
      rn2p *= 1.f / (kRScale * kRScale);
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
        // the QJL GEMM of tile t - 1 has consumed the residual operand once its projection
        // is complete: collect those signs, then hand over this tile's residual
        if (t >= 1) {
          if (!wait(z_full, (uint32_t)((t - 1) & 1))) { fail(106); ok = false; break; }
          take_signs();
        }
        const uint32_t rz = lane_base + kColR + c0 / 2;
        if constexpr (CQ == 32) {
          tmem_st16(rz, hi);
          tmem_st16(rz + D / 2, lo);
        } else {
          tmem_st8(rz, hi);
          tmem_st8(rz + D / 2, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(r_full);
        s_rn[(b * 4 + wg) * kTileM + row] = rn2p;
        mbar_arrive(xr + b);
        if (t >= 1 && !finish(t - 1)) { ok = false; break; }
#pragma unroll
        for (int p = 0; p < PW; ++p) pend_words[p] = words[p];
        pend_n = nrm;
        pend_v = v;
      } else {
        store_quarter(t, v, words, nrm, 0.f);
      }
    }
    if (PROD && ok && nloc >= 1) {
      if (wait(z_full, (uint32_t)((nloc - 1) & 1))) {
        take_signs();
        finish(nloc - 1);
      } else {
        fail(106);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
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
  a.cap = dst->cap;
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
  cudaError_t e = ensure_smem_attrs<quantize_tc_kernel<D, PROD, K>>(smem_bytes, false);
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

// The fused kernel's shapes: bf16 input with 16-byte aligned rows, d in {64, 128}, at least
// one 128-row tile (the workspace path takes every other call).
bool quantize_tc_applies(const tq_ctx* ctx, int x_dtype, int64_t n, int64_t ld) {
  const int d = ctx->lay.d, k = ctx->lay.k;
  const bool prod = ctx->mode == TQ_MODE_PROD;
  const bool built = prod ? (k >= 1 && k <= 3) : (k >= 2 && k <= 4);   // the instantiated code widths
  return built && x_dtype == TQ_DTYPE_BF16 && ctx->Pi_split && (d == 64 || d == 128) && (ld * 2) % 16 == 0 &&
         n >= kTileM;
}

int launch_quantize_tc(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const tq_packed* dst,
                       const int64_t* slots, cudaStream_t st) {
  if (!quantize_tc_applies(ctx, x_dtype, n, ld) || (reinterpret_cast<uintptr_t>(x) % 16) != 0) return kNotHandled;
  const int d = ctx->lay.d, k = ctx->lay.k;
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
