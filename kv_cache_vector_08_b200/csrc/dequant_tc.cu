// Dequantize on the 5th-generation tensor cores (tcgen05, A operand in TMEM, B staged by TMA).
//
// turboquant.net "Quant / DeQuant 函数": the MSE reconstruction of a stored vector is
// x_hat = ||x|| Pi^T c[idx].  For a tile of 128 stored vectors that is one dense product
//
//   D [128 x N] = C [128 x K] * (16 Pi^T)^T        C[v][j] = c[idx_vj] (zero for j >= d)
//   x_hat[v][i] = norm_v / 16 * D[v][i]
//
// with K = d_pad (32-coordinate code groups) and N = 16 ceil(d / 16).  C is held as fp16
// hi + lo and 16 Pi^T as fp16 hi + lo; the three products hi*hi + hi*lo + lo*hi carry
// about 22 bits, so x_hat is fp32-accurate well inside the 1e-3 + 2e-3 |x| contract.
//
// Roles (one persistent CTA per SM, 320 threads): warp 0 loads the two B splits once by
// TMA; warp 1 owns TMEM and issues the MMAs; warps 2-9 are workers.  A worker owns one
// vector row (its TMEM lane) and half of the code groups / output columns: it loads the
// row's packed code words one tile ahead, turns every code into the fp16 hi / lo pair of
// its centroid with one table lookup, writes them into its lane of the A buffer with
// tcgen05.st, and after the MMAs reads the row's accumulator back (tcgen05.ld), scales it
// by the stored norm and writes it out.  TMEM holds two accumulators and two A buffers
// (hi and lo halves), so the decode of tile t+1 and the MMAs of tile t overlap with the
// epilogue of tile t-1.  Every wait is bounded; a timeout records an error code in the
// context's error word and the CTA winds down.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_ops.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;
using mmaops::prmt;

constexpr int kDqTile = 128;
constexpr int kDqWorkerWarps = 8;
constexpr int kDqWorkers = 32 * kDqWorkerWarps;
constexpr int kDqThreads = 64 + kDqWorkers;
constexpr uint64_t kDqWaitNs = 2000000000ull;
constexpr uint32_t kDqCols = 512;    // D[2] at columns 0, 128; A[2] at 256, 384 (hi at +0, lo at +64)
constexpr float kDqBScale = 16.f;    // B holds 16 Pi^T (keeps the small entries of Pi normal in fp16)

struct DqArgs {
  const uint8_t* codes;
  const uint16_t* norm;
  const uint16_t* rnorm;     // QJL-augmented reconstruction: residual norms
  const int64_t* slots;
  float* out;
  int64_t n, ld;
  int d, code_bytes;
  int vec4;             // out rows start 16-byte aligned: float4 stores
  int64_t cap;          // slots in the packed storage (a gathered slot outside [0, cap) is skipped)
  uint64_t wait_ns;     // limit of the pipeline waits
  int stall;            // test hook: the MMA issuer first waits on a barrier nothing arrives on
  uint32_t tbl[32];     // P-bit code -> fp16 hi (bits 0-15) | fp16 lo (bits 16-31) of its centroid
  // 4-bit codes: byte tables indexed by the low 3 code bits (8 entries = 2 registers each):
  // low / high bytes of the fp16 hi and lo parts; in MSE mode the entries are the
  // magnitudes and the top (sign) bit is applied separately, in prod mode they are signed
  uint32_t bt[4][2];
  int mse_sign;         // 1: MSE mode (apply the top bit as the sign)
  int* err;
};

template <int NG, bool QJL>
struct DqSmem {
  static constexpr int K = 32 * NG;
  static constexpr int KA = (K + 63) / 64;                 // 128-byte K atoms per row
  static constexpr int NMAX = K;                           // N <= K
  static constexpr int SPLIT = KA * NMAX * 128;            // one B split
  static constexpr int OFF_B = 0;                          // 16 Pi^T hi, lo (then 16 kappa S^T hi, lo)
  static constexpr int OFF_TBL = OFF_B + (QJL ? 4 : 2) * SPLIT;
  static constexpr int OFF_BAR = OFF_TBL + 32 * 4;
  static constexpr int BYTES = OFF_BAR + 256 + 1024;       // + barriers, + alignment slack
};

template <int NG, int P, bool QJL>
__global__ void __launch_bounds__(kDqThreads, 1) dequant_tc_kernel(const __grid_constant__ CUtensorMap tm_b,
                                                                   const __grid_constant__ CUtensorMap tm_s,
                                                                   const int N, const DqArgs A) {
  using SM = DqSmem<NG, QJL>;
  // A buffers in TMEM: two (hi at +0, lo at +64) for the plain reconstruction; one (hi,
  // lo, +-||r|| at +128) for the QJL-augmented one
  constexpr int NA = QJL ? 1 : 2;
  constexpr int K = SM::K, KA = SM::KA, NK = K / 16;
  constexpr int G0 = (NG + 1) / 2;       // code groups of half 0 (half 1 takes the rest)
  constexpr int PW = G0 * P;             // code words a worker holds per tile
  extern __shared__ uint8_t dq_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dq_smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* s_tbl = reinterpret_cast<uint32_t*>(smem + SM::OFF_TBL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);
  uint64_t* b_full = bars;          // B splits landed
  uint64_t* a_full = bars + 1;      // [2] workers -> MMA: A buffer written
  uint64_t* a_empty = bars + 3;     // [2] MMA -> workers: A buffer consumed
  uint64_t* d_full = bars + 5;      // [2] MMA -> workers: accumulator ready
  uint64_t* d_empty = bars + 7;     // [2] workers -> MMA: accumulator read
  uint64_t* drain = bars + 9;       // every issued MMA complete
  uint64_t* never = bars + 10;      // test hook: no thread ever arrives here
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (A.n + kDqTile - 1) / kDqTile;
  const int nloc = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

  if (threadIdx.x == 0) {
    mbar_init(b_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(a_full + b, kDqWorkers);
      mbar_init(a_empty + b, 1);
      mbar_init(d_full + b, 1);
      mbar_init(d_empty + b, kDqWorkers);
    }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 32) s_tbl[threadIdx.x] = A.tbl[threadIdx.x];
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDqCols);
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
  auto wait = [&](uint64_t* bar, uint32_t parity) { return mbar_wait(bar, parity, abort_v, A.wait_ns); };

  if (warp == 0) {
    // ------------------------------------------------------------- B loader (once)
    if (lane == 0) {
      prefetch_tensormap(&tm_b);
      mbar_arrive_expect_tx(b_full, (uint32_t)((QJL ? 4 : 2) * KA * N * 128));
      for (int s = 0; s < 2; ++s)
        for (int a = 0; a < KA; ++a) tma_load_2d(smem + SM::OFF_B + s * SM::SPLIT + a * N * 128, &tm_b, 64 * a, s * N, b_full);
      if (QJL)
        for (int s = 0; s < 2; ++s)
          for (int a = 0; a < KA; ++a)
            tma_load_2d(smem + SM::OFF_B + (2 + s) * SM::SPLIT + a * N * 128, &tm_s, 64 * a, s * N, b_full);
      mbar_wait(b_full, 0, nullptr, kDqWaitNs);   // the copies land before the CTA can exit
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kDqTile, N, 0);
      const uint32_t b_addr = smem_u32(smem + SM::OFF_B);
      bool ok = true;
      if (A.stall && !wait(never, 0)) { fail(305); ok = false; }   // the injected stall runs out
      if (ok && !wait(b_full, 0)) { fail(301); ok = false; }
      for (int t = 0; ok && t < nloc; ++t) {
        const int b = t & 1, ab = t % NA;
        const uint32_t ph = (uint32_t)((t >> 1) & 1), aph = (uint32_t)((t / NA) & 1);
        if (!wait(a_full + ab, aph) || !wait(d_empty + b, ph ^ 1)) { fail(302); break; }
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(b * 128), acol = tmem + 256u + (uint32_t)(ab * 128);
        // (A split, B split): C hi * Pi hi, C hi * Pi lo, C lo * Pi hi; then, QJL-augmented,
        // (+-||r||) * (kappa S)^T hi and lo
        for (int sp = 0; sp < (QJL ? 5 : 3); ++sp) {
          const uint32_t a_split = acol + (sp == 2 ? 64u : sp >= 3 ? 128u : 0u);
          const int b_split = sp == 1 ? 1 : sp == 3 ? 2 : sp == 4 ? 3 : 0;
          for (int ks = 0; ks < NK; ++ks) {
            const uint64_t db = desc_sw128(b_addr + b_split * SM::SPLIT + (ks >> 2) * N * 128 + (ks & 3) * 32);
            mma_ts(dcol, a_split + (uint32_t)(ks * 8), db, idesc, (sp | ks) ? 1u : 0u);
          }
        }
        mma_commit(a_empty + ab);
        mma_commit(d_full + b);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kDqWaitNs);
    }
  } else {
    // ---------------------------------------------------------------------- workers
    const int wq = warp & 3, half = (warp - 2) >> 2;
    const int row = wq * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const int g_lo = half ? G0 : 0, g_hi = half ? NG : G0;
    const int nch = N / 16, c0 = (nch + 1) / 2;
    const int ch_lo = half ? c0 : 0, ch_hi = half ? nch : c0;
    auto load_row = [&](int t, uint32_t (&w)[PW], float& nrm, int64_t& v, uint32_t& rb) {
      const int64_t tile = blockIdx.x + (int64_t)t * gridDim.x;
      v = tile * kDqTile + row;
#pragma unroll
      for (int i = 0; i < PW; ++i) w[i] = 0u;
      nrm = 0.f;
      rb = 0u;
      if (t < nloc && v < A.n) {
        const int64_t slot = A.slots ? __ldg(A.slots + v) : v;
        if (slot < 0 || slot >= A.cap) {        // out of range: zeros, and the error word says so
          if (A.err) atomicCAS(A.err, 0, (int)kErrSlotRange);
          return;
        }
        const uint32_t* rec = reinterpret_cast<const uint32_t*>(A.codes + slot * (int64_t)A.code_bytes);
#pragma unroll
        for (int g = 0; g < G0; ++g)
          if (g_lo + g < g_hi)
#pragma unroll
            for (int p = 0; p < P; ++p) w[g * P + p] = __ldg(rec + (g_lo + g) * P + p);
        nrm = __half2float(__ushort_as_half(__ldg(A.norm + slot)));
        if (QJL) rb = (uint32_t)__ldg(A.rnorm + slot) & 0x7FFFu;
      }
    };
    uint32_t cur[PW], nxt[PW];
    float cur_n, nxt_n, pend_n = 0.f;
    int64_t cur_v, nxt_v, pend_v = -1;
    uint32_t cur_r, nxt_r;
    load_row(0, cur, cur_n, cur_v, cur_r);
    bool ok = true;
    // epilogue of local tile t: accumulator -> registers -> scaled rows of out
    auto epilogue = [&](int t, float nrm, int64_t v) -> bool {
      const int b = t & 1;
      if (!wait(d_full + b, (uint32_t)((t >> 1) & 1))) { fail(303); return false; }
      tc_fence_after();
      // all of the row's column chunks are requested before one wait (one TMEM round trip)
      uint32_t r[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (ch_lo + c < ch_hi) tmem_ld16(lane_base + (uint32_t)(b * 128 + 16 * (ch_lo + c)), r[c]);
      tmem_ld_wait();
      float acc[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[c][i] = __uint_as_float(r[c][i]);
      tc_fence_before();
      mbar_arrive(d_empty + b);
      if (v < A.n) {
        const float s = nrm * (1.f / kDqBScale);
        float* o = A.out + v * A.ld;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = 16 * (ch_lo + c);
          if (ch_lo + c >= ch_hi) continue;
          if (A.vec4 && col + 16 <= A.d) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(o + col + i) =
                  make_float4(acc[c][i] * s, acc[c][i + 1] * s, acc[c][i + 2] * s, acc[c][i + 3] * s);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (col + i < A.d) o[col + i] = acc[c][i] * s;
          }
        }
      }
      return true;
    };
    for (int t = 0; t < nloc; ++t) {
      const int ab = t % NA;
      load_row(t + 1, nxt, nxt_n, nxt_v, nxt_r);       // one tile ahead: its loads fly during this tile
      // codes -> fp16 (hi, lo) pairs of the centroids, two coordinates per 32-bit column, of
      // this worker's group g (and, QJL, the fp16 +-||r|| pairs)
      auto convert = [&](int g, uint32_t (&hi)[16], uint32_t (&lo)[16], uint32_t (&sg)[16]) {
        if constexpr (P == 4) {
          // 4-bit codes: slice u of a group is word u, coordinate j of the slice has its low
          // three code bits in nibble j and its top bit at the msb of byte j (j < 4) or, after
          // a shift by 4, of byte j - 4; one byte permute looks up four bytes
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t w = cur[g * P + u];
            const uint32_t sel = w & 0x77777777u;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t sl = hh ? sel >> 16 : sel;
              const uint32_t top = hh ? w << 4 : w;        // top bits at byte msbs
              const uint32_t sgn = A.mse_sign ? (top & 0x80808080u) : 0u;
              const uint32_t hl = prmt(A.bt[0][0], A.bt[0][1], sl), hh8 = prmt(A.bt[1][0], A.bt[1][1], sl) ^ sgn;
              const uint32_t ll = prmt(A.bt[2][0], A.bt[2][1], sl), lh8 = prmt(A.bt[3][0], A.bt[3][1], sl) ^ sgn;
              const int i = 4 * u + 2 * hh;                // pair index of coordinates 8u + 4hh, +1
              hi[i] = prmt(hl, hh8, 0x5140u);
              hi[i + 1] = prmt(hl, hh8, 0x7362u);
              lo[i] = prmt(ll, lh8, 0x5140u);
              lo[i + 1] = prmt(ll, lh8, 0x7362u);
              if constexpr (QJL) {
                const uint32_t nm = ~top;                  // fp16 sign set where the QJL bit is 0
                sg[i] = (prmt(nm, 0u, 0x1404u) & 0x80008000u) | (cur_r | (cur_r << 16));
                sg[i + 1] = (prmt(nm, 0u, 0x3424u) & 0x80008000u) | (cur_r | (cur_r << 16));
              }
            }
          }
          // coordinates >= d are zero
          const int j0 = 32 * (g_lo + g);
          if (j0 + 32 > A.d) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (j0 + e >= A.d) {
                const uint32_t keep = (e & 1) ? 0x0000FFFFu : 0xFFFF0000u;
                hi[e / 2] &= keep;
                lo[e / 2] &= keep;
                if constexpr (QJL) sg[e / 2] &= keep;
              }
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int j = 32 * (g_lo + g) + e;
            const uint32_t ca = group_code(cur + g * P, P, e), cb = group_code(cur + g * P, P, e + 1);
            const uint32_t ta = (j < A.d) ? s_tbl[ca] : 0u;
            const uint32_t tb = (j + 1 < A.d) ? s_tbl[cb] : 0u;
            hi[e / 2] = __byte_perm(ta, tb, 0x5410);
            lo[e / 2] = __byte_perm(ta, tb, 0x7632);
            if constexpr (QJL) {
              // +-||r|| (fp16; the sign bit set where the QJL sign bit is 0), zero past d
              const uint32_t sa = (j < A.d) ? (cur_r | ((((ca >> (P - 1)) & 1u) ^ 1u) << 15)) : 0u;
              const uint32_t sb = (j + 1 < A.d) ? (cur_r | ((((cb >> (P - 1)) & 1u) ^ 1u) << 15)) : 0u;
              sg[e / 2] = sa | (sb << 16);
            }
          }
        }
      };
      const uint32_t acol = lane_base + 256u + (uint32_t)(ab * 128);
      if constexpr (!QJL) {
        // all groups converted before the wait for the A buffer (the conversion overlaps the
        // MMAs of the tile before)
        uint32_t hi[G0][16], lo[G0][16], sg0[16];
#pragma unroll
        for (int g = 0; g < G0; ++g) convert(g, hi[g], lo[g], sg0);
        if (!wait(a_empty + ab, (uint32_t)(((t / NA) & 1) ^ 1))) { fail(304); ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < G0; ++g) {
          if (g_lo + g < g_hi) {
            tmem_st16(acol + (uint32_t)(16 * (g_lo + g)), hi[g]);
            tmem_st16(acol + 64u + (uint32_t)(16 * (g_lo + g)), lo[g]);
          }
        }
      } else {
        // QJL: three operand halves per group would not fit in registers for every group at
        // once, so each group is converted and stored in turn after the wait
        if (!wait(a_empty + ab, (uint32_t)(((t / NA) & 1) ^ 1))) { fail(304); ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < G0; ++g) {
          if (g_lo + g < g_hi) {
            uint32_t hi[16], lo[16], sg[16];
            convert(g, hi, lo, sg);
            tmem_st16(acol + (uint32_t)(16 * (g_lo + g)), hi);
            tmem_st16(acol + 64u + (uint32_t)(16 * (g_lo + g)), lo);
            tmem_st16(acol + 128u + (uint32_t)(16 * (g_lo + g)), sg);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(a_full + ab);
      if (t >= 1 && !epilogue(t - 1, pend_n, pend_v)) { ok = false; break; }
      pend_n = cur_n;
      pend_v = cur_v;
#pragma unroll
      for (int i = 0; i < PW; ++i) cur[i] = nxt[i];
      cur_n = nxt_n;
      cur_v = nxt_v;
      cur_r = nxt_r;
    }
    if (ok && nloc >= 1) epilogue(nloc - 1, pend_n, pend_v);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDqCols);
  }
}

template <int NG, int P, bool QJL>
int launch_dq_t(const CUtensorMap& tmb, const CUtensorMap& tms, int N, const DqArgs& a, int64_t n, int dev,
                cudaStream_t st) {
  using SM = DqSmem<NG, QJL>;
  auto kern = dequant_tc_kernel<NG, P, QJL>;
  // one CTA per SM (it owns all 512 TMEM columns): ask for more than half the shared memory
  const int smem_bytes = SM::BYTES > 120 * 1024 ? SM::BYTES : 120 * 1024;
  cudaError_t e = ensure_smem_attrs<dequant_tc_kernel<NG, P, QJL>>(smem_bytes, false);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(dequant_tc)");
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (n + kDqTile - 1) / kDqTile;
  const int grid = (int)std::min<int64_t>(ntiles, sms);
  kern<<<grid, kDqThreads, smem_bytes, st>>>(tmb, tms, N, a);
  count_launch();
  return check_launch("dequant_tc_kernel");
}

}  // namespace

// x_hat = norm * Pi^T c[idx] (qjl: + norm sqrt(pi/2)/m rnorm S^T (2 s - 1)) of n stored
// vectors on the tensor cores (d <= 128).
int launch_dequantize_tc(const tq_ctx* ctx, const tq_packed* src, const int64_t* slots, int64_t n, float* out,
                         int64_t ld, bool qjl, cudaStream_t st) {
  const int d = ctx->lay.d;
  if (d > 128 || !ctx->PiT_f16) return fail(TQ_ERR_UNSUPPORTED, "tq_dequantize supports d <= 128");
  if (qjl && (ctx->mode != TQ_MODE_PROD || !ctx->ST_f16))
    return fail(TQ_ERR_INVALID_ARG, "the QJL-augmented reconstruction needs a prod-mode context");
  if (n == 0) return TQ_OK;
  const int NG = ctx->lay.d_pad / 32, K = ctx->lay.d_pad, N = 16 * ((d + 15) / 16);
  CUtensorMap tmb, tms;
  if (!make_map(&tmb, ctx->PiT_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)N, (uint64_t)K, (uint64_t)K * 2,
                (uint32_t)N))
    return fail(TQ_ERR_INTERNAL, "tensor map for the dequantize operand");
  tms = tmb;
  if (qjl && !make_map(&tms, ctx->ST_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)N, (uint64_t)K,
                       (uint64_t)K * 2, (uint32_t)N))
    return fail(TQ_ERR_INTERNAL, "tensor map for the QJL operand");
  DqArgs a{};
  a.codes = src->codes;
  a.norm = src->norm;
  a.rnorm = src->rnorm;
  a.slots = slots;
  a.out = out;
  a.n = n;
  a.ld = ld;
  a.d = d;
  a.code_bytes = ctx->lay.code_bytes;
  a.vec4 = ((reinterpret_cast<uintptr_t>(out) & 15) == 0 && (ld & 3) == 0) ? 1 : 0;
  a.err = ctx->dev_err;
  a.cap = src->cap;
  a.wait_ns = pipeline_wait_ns();
  a.stall = debug_stall() ? 1 : 0;
  const int k = ctx->lay.k, P = ctx->lay.planes;
  for (int code = 0; code < 32; ++code) {
    uint32_t v = 0;
    if (code < (1 << P)) {
      const double c = ctx->host.centroids[code_index((uint32_t)code & ((1u << k) - 1u), k)];
      const __half h = __float2half_rn((float)c);
      const __half l = __float2half_rn((float)(c - (double)__half2float(h)));
      v = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    }
    a.tbl[code] = v;
  }
  if (P == 4) {
    // 8-entry byte tables over the low three code bits (MSE: magnitude rank; prod: sign flag
    // and magnitude rank), for the fp16 hi and lo parts of the centroid
    const bool mse = ctx->mode == TQ_MODE_MSE;
    a.mse_sign = mse ? 1 : 0;
    uint8_t b[4][8];
    for (int c3 = 0; c3 < 8; ++c3) {
      const double c = mse ? ctx->host.centroids[(1 << (k - 1)) + c3] : ctx->host.centroids[code_index((uint32_t)c3, k)];
      const __half h = __float2half_rn((float)c);
      const __half l = __float2half_rn((float)(c - (double)__half2float(h)));
      const uint16_t hb = __half_as_ushort(h), lb = __half_as_ushort(l);
      b[0][c3] = (uint8_t)(hb & 0xFF);
      b[1][c3] = (uint8_t)(hb >> 8);
      b[2][c3] = (uint8_t)(lb & 0xFF);
      b[3][c3] = (uint8_t)(lb >> 8);
    }
    for (int t = 0; t < 4; ++t)
      for (int r = 0; r < 2; ++r)
        a.bt[t][r] = b[t][4 * r] | (b[t][4 * r + 1] << 8) | (b[t][4 * r + 2] << 16) | ((uint32_t)b[t][4 * r + 3] << 24);
  }
  const int dev = ctx->device;
#define TQ_DQ_CASE(GG, PP) \
  if (NG == GG && P == PP) {                                                                  \
    if (qjl) return launch_dq_t<GG, PP, true>(tmb, tms, N, a, n, dev, st);                    \
    return launch_dq_t<GG, PP, false>(tmb, tms, N, a, n, dev, st);                            \
  }
#define TQ_DQ_G(GG) TQ_DQ_CASE(GG, 1) TQ_DQ_CASE(GG, 2) TQ_DQ_CASE(GG, 3) TQ_DQ_CASE(GG, 4) TQ_DQ_CASE(GG, 5)
  TQ_DQ_G(1) TQ_DQ_G(2) TQ_DQ_G(3) TQ_DQ_G(4)
#undef TQ_DQ_G
#undef TQ_DQ_CASE
  return fail(TQ_ERR_INTERNAL, "dequantize: no kernel for this code layout");
}

}  // namespace tq
