// Quantize any width d and any input type on the tensor cores, through a workspace.
//
// turboquant.net "Quant / DeQuant 函数" (y = Pi x / ||x||, nearest Lloyd-Max centroid per
// coordinate), "残差 norm 存储" (||r|| as one fp16), admirer.cn QJL paragraph (signs of S r).
// The fused bf16 kernel (quantize_tc.cu) keeps Pi and M resident in shared memory, which
// bounds it to d <= 128 with exact bf16 input.  This path covers every other shape (fp32 /
// fp16 input, the search widths d = 200, 1536, 3072, batches below one tile) with three
// kernels over a workspace of row chunks:
//
//   prep       one warp per row: ||x|| in float64, fp16 norm out, a power-of-two row scale
//              2^s (max |x| 2^s in [2^14, 2^15)) and the row as fp16 hi + lo of x 2^s
//              (exact to ~2^-22, zero padded to K = 64 ceil(d/64) columns)
//   project    tcgen05 GEMM, D [128 x Nb] = X [128 x K] (16 Pi)^T over K atoms staged by
//              TMA, as hi*hi + hi*lo + lo*hi fp16 products (fp32-accurate to ~2^-22);
//              epilogue (thread = row, 32 columns = one code group at a time): y = D / (16
//              2^s ||x||), sign-magnitude index codes by comparison with the codebook's
//              positive boundaries, the index bits of the group's P code words, r = y -
//              c[idx] as fp16 hi + lo of 2^8 r into the workspace, ||r||^2 partials
//   sign       (prod mode) the same GEMM on A = 2^8 r, B = 16 M (M = S Pi^T, so M r = S (u -
//              Pi^T c[idx])); epilogue: QJL sign bits [z >= 0] ORed into the code words,
//              rnorm = fp16(sqrt(sum of the partials))
//
// Work unit of the GEMMs = (128-row tile, N block of <= 256 output columns), N blocks of
// a tile on consecutive units so the tile's A atoms are re-read from L2.  Roles per CTA
// (persistent, one per SM): warp 0 TMA producer (2 stages of A hi/lo + B hi/lo atoms),
// warp 1 TMEM owner and MMA issuer, warps 2-17 epilogue (thread = row x 64 columns).
// Precision: the tensor core adds each instruction's products into its fp32 accumulator
// with a directed rounding, so over thousands of accumulation steps the error grows
// linearly (d = 1536: ~1e-5 relative, far above the 1e-6 decision band).  Each 64-column
// K atom (12 MMAs: 3 split products x 4 k-steps) therefore starts a fresh accumulator in
// one of two TMEM buffers, and the epilogue threads add the atom partials into fp32
// registers (round to nearest) as the MMAs of the next atom run.  Every wait is bounded;
// a timeout records an error code in the context's error word and the CTA winds down.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

constexpr int kGenTile = 128;
constexpr int kGenNb = 256;                       // widest N block (accumulator columns)
constexpr int kGenStages = 2;
constexpr int kGenEpiWarps = 16;                  // 4 per TMEM lane quarter, 64 columns each
constexpr int kGenThreads = 64 + 32 * kGenEpiWarps;  // + TMA warp, MMA warp
constexpr uint64_t kGenWaitNs = 2000000000ull;
constexpr int64_t kGenChunk = 131072;             // rows per workspace chunk
constexpr float kGenRScale = 256.f;               // the residual enters the sign GEMM as 2^8 r
constexpr float kGenBScale = 16.f;                // B operands hold 16 Pi and 16 M

// Per-row values the prep kernel leaves for the GEMM epilogues.
struct RowInfo {
  float inv;    // 1 / (16 * 2^s * ||x||), 0 for a zero row
  float nrm;    // ||x|| (fp32)
};

struct GenLayout {
  int K, N, NB;              // MMA K (64-multiple), output columns (d_pad), N blocks
  int64_t rows;              // rows per chunk (a multiple of 128)
  size_t off_x, off_r, off_info, off_rn2, total;
};

GenLayout gen_layout(const tq_ctx* ctx, int64_t n) {
  GenLayout L{};
  const int d = ctx->lay.d;
  L.K = 64 * ((d + 63) / 64);
  L.N = ctx->lay.d_pad;
  L.NB = (L.N + kGenNb - 1) / kGenNb;
  const int64_t want = std::min<int64_t>(std::max<int64_t>(n, 1), kGenChunk);
  L.rows = (want + kGenTile - 1) / kGenTile * kGenTile;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t xb = (size_t)2 * L.rows * L.K * sizeof(__half);
  L.off_x = 0;
  L.off_r = up(xb);
  L.off_info = L.off_r + (ctx->mode == TQ_MODE_PROD ? up(xb) : 0);
  L.off_rn2 = L.off_info + up((size_t)L.rows * sizeof(RowInfo));
  L.total = L.off_rn2 + up((size_t)L.rows * L.NB * 4 * sizeof(float));
  return L;
}

// ------------------------------------------------------------------------------ prep
template <typename T>
__device__ __forceinline__ float load_elem(const T* p) {
  if constexpr (std::is_same<T, float>::value) return __ldg(p);
  else if constexpr (std::is_same<T, __half>::value) return __half2float(*p);
  else return __bfloat162float(*p);
}

struct PrepArgs {
  const void* x;
  const int32_t* cols;       // element j of a row is x[row * ld + cols[j]] (NULL: x[row * ld + j])
  int64_t ld, n, row0;       // rows row0 .. row0+n of x form this chunk
  int d, K;
  const int64_t* slots;      // global row -> slot (NULL: the row itself)
  uint16_t* norm;
  __half* X;                 // hi [lo_off][K], then lo [lo_off][K]
  __half* R;                 // residual operand (prod mode; same layout), or NULL
  int N;                     // columns the projection epilogue writes into R (d_pad)
  int64_t rows, lo_off;      // rows written (n rounded up to the tile), row offset of lo
  int64_t cap;               // slots in the packed storage
  RowInfo* info;
  int* err;
};

template <typename T>
__global__ void __launch_bounds__(256) quantize_prep_kernel(PrepArgs A) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + warp;     // row within the chunk
  if (r >= A.rows) return;
  __half* xh = A.X + r * A.K;
  __half* xl = A.X + (A.lo_off + r) * A.K;
  if (A.R) {                 // residual columns [N, K) are never written by the epilogue: zeros
    for (int i = A.N + lane; i < A.K; i += 32) {
      A.R[r * A.K + i] = __float2half(0.f);
      A.R[(A.lo_off + r) * A.K + i] = __float2half(0.f);
    }
  }
  if (r >= A.n) {            // padding rows of the last tile: zeros
    for (int i = lane; i < A.K; i += 32) {
      xh[i] = __float2half(0.f);
      xl[i] = __float2half(0.f);
    }
    return;
  }
  const int64_t v = A.row0 + r;
  const T* x = static_cast<const T*>(A.x) + v * A.ld;
  double s2 = 0.0;
  float mx = 0.f;
  bool bad_col = false;
  auto col = [&](int i) -> int {               // column of element i (out-of-range entries read as 0)
    if (!A.cols) return i;
    const int c = A.cols[i];
    if (c < 0 || c >= A.ld) { bad_col = true; return -1; }
    return c;
  };
  for (int i = lane; i < A.d; i += 32) {
    const int c = col(i);
    const float e = c >= 0 ? load_elem(x + c) : 0.f;
    s2 = fma((double)e, (double)e, s2);
    mx = fmaxf(mx, fabsf(e));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const double nrm = sqrt(s2);
  // 2^s with max |x| 2^s in [2^14, 2^15): fp16 hi + lo then hold x 2^s to ~2^-22
  int e2 = 0;
  if (mx > 0.f) frexpf(mx, &e2);                        // mx = f 2^e2, f in [0.5, 1)
  const float scale = mx > 0.f ? ldexpf(1.f, 15 - e2) : 1.f;
  for (int i = lane; i < A.K; i += 32) {
    const int c = i < A.d ? col(i) : -1;
    const float e = c >= 0 ? load_elem(x + c) * scale : 0.f;
    const __half h = __float2half_rn(e);
    xh[i] = h;
    xl[i] = __float2half_rn(e - __half2float(h));
  }
  if (bad_col && A.err) atomicCAS(A.err, 0, (int)kErrPermRange);
  if (lane == 0) {
    const int64_t slot = A.slots ? A.slots[v] : v;
    if (slot < 0 || slot >= A.cap) {        // out of range: the row is skipped (the GEMMs skip it too)
      if (A.err) atomicCAS(A.err, 0, (int)kErrSlotRange);
    } else {
      A.norm[slot] = __half_as_ushort(__double2half(nrm));
    }
    RowInfo ri;
    ri.nrm = (float)nrm;
    ri.inv = nrm > 0.0 ? (float)(1.0 / ((double)kGenBScale * (double)scale * nrm)) : 0.f;
    A.info[r] = ri;
  }
}

// ------------------------------------------------------------------------------ GEMM
struct GemmArgs {
  int64_t n, rows, row0;     // valid rows of the chunk, rows processed (tile multiple), first global row
  int64_t lo_off;            // row offset of the lo halves in the A and R buffers
  int K, N, NB, d, code_bytes;
  int box_b;                 // rows of a B box (min(256, N)): bytes a B load always delivers
  const int64_t* slots;
  uint8_t* codes;
  uint16_t* rnorm;
  const RowInfo* info;
  __half* R;                 // [2][rows][K] (project epilogue output, prod mode)
  float* rn2;                // [rows][NB][4] (one partial per 64-column part)
  float pos_t[8];            // positive boundaries above 0, ascending (+inf beyond)
  float mag[8];              // centroid magnitudes c[K/2 + m]
  int64_t cap;               // slots in the packed storage
  uint64_t wait_ns;          // limit of the pipeline waits
  int* err;
};

template <int P, int KB, bool PROD, bool SIGN>
__global__ void __launch_bounds__(kGenThreads, 1) quantize_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                                       const __grid_constant__ CUtensorMap tm_b,
                                                                       const GemmArgs A) {
  constexpr int STAGE_A = kGenTile * 128;               // one 128-row x 64-column fp16 atom
  constexpr int STAGE_B = kGenNb * 128;
  constexpr int STAGE = 2 * STAGE_A + 2 * STAGE_B;
  constexpr int LEVELS = 1 << KB;
  extern __shared__ uint8_t gen_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gen_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGenStages * STAGE);
  uint64_t* full = bars;                      // [stages] TMA -> MMA
  uint64_t* empty = bars + kGenStages;        // [stages] MMA -> TMA
  uint64_t* acc_full = bars + 2 * kGenStages; // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;         // [2] epilogue -> MMA
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KA = A.K / 64;
  const int64_t units = (A.rows / kGenTile) * A.NB;
  const int nloc = (int)((units - blockIdx.x + gridDim.x - 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGenStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 32 * kGenEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
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
  auto unit_of = [&](int t, int64_t& mt, int& nb, int& width) {
    const int64_t u = blockIdx.x + (int64_t)t * gridDim.x;
    mt = u / A.NB;
    nb = (int)(u % A.NB);
    width = min(kGenNb, A.N - nb * kGenNb);
  };

  if (warp == 0) {
    // ----------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_a);
      prefetch_tensormap(&tm_b);
      int pending[kGenStages];
      for (int s = 0; s < kGenStages; ++s) pending[s] = -1;
      int64_t q = 0;
      bool ok = true;
      for (int t = 0; ok && t < nloc; ++t) {
        int64_t mt;
        int nb, width;
        unit_of(t, mt, nb, width);
        for (int a = 0; a < KA; ++a, ++q) {
          const int s = (int)(q % kGenStages);
          const uint32_t ph = (uint32_t)((q / kGenStages) & 1);
          if (!wait(empty + s, ph ^ 1)) { fail(401); ok = false; break; }
          uint8_t* st = smem + s * STAGE;
          mbar_arrive_expect_tx(full + s, (uint32_t)(2 * STAGE_A + 2 * A.box_b * 128));
          tma_load_2d(st, &tm_a, 64 * a, (int)(mt * kGenTile), full + s);
          tma_load_2d(st + STAGE_A, &tm_a, 64 * a, (int)(A.lo_off + mt * kGenTile), full + s);
          tma_load_2d(st + 2 * STAGE_A, &tm_b, 64 * a, nb * kGenNb, full + s);
          tma_load_2d(st + 2 * STAGE_A + STAGE_B, &tm_b, 64 * a, A.N + nb * kGenNb, full + s);
          pending[s] = (int)ph;
        }
      }
      for (int s = 0; s < kGenStages; ++s)
        if (pending[s] >= 0) mbar_wait(full + s, (uint32_t)pending[s], nullptr, kGenWaitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t q = 0;
      bool ok = true;
      for (int t = 0; ok && t < nloc; ++t) {
        int64_t mt;
        int nb, width;
        unit_of(t, mt, nb, width);
        const uint32_t idesc = idesc_f16(kGenTile, width, 0);
        for (int a = 0; a < KA; ++a, ++q) {
          // atom q into accumulator buffer q & 1, from zero
          const int b = (int)(q & 1);
          if (!wait(acc_empty + b, (uint32_t)(((q >> 1) & 1) ^ 1))) { fail(402); ok = false; break; }
          const int s = (int)(q % kGenStages);
          if (!wait(full + s, (uint32_t)((q / kGenStages) & 1))) { fail(403); ok = false; break; }
          tc_fence_after();
          const uint32_t dcol = tmem + (uint32_t)(b * kGenNb);
          const uint32_t base = smem_u32(smem + s * STAGE);
          // (A split, B split): hi*hi, hi*lo, lo*hi
          for (int sp = 0; sp < 3; ++sp) {
            const uint32_t aa = base + (sp == 2 ? STAGE_A : 0);
            const uint32_t bb = base + 2 * STAGE_A + (sp == 1 ? STAGE_B : 0);
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(dcol, desc_sw128(aa + kk * 32), desc_sw128(bb + kk * 32), idesc, (sp | kk) ? 1u : 0u);
          }
          mma_commit(empty + s);
          mma_commit(acc_full + b);
        }
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kGenWaitNs);
    }
  } else {
    // --------------------------------------------------------------------- epilogue
    const int wq = warp & 3, part = (warp - 2) >> 2;      // lane quarter, 64-column part
    const int row = wq * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    int64_t q = 0;
    bool ok = true;
    for (int t = 0; ok && t < nloc; ++t) {
      int64_t mt;
      int nb, width;
      unit_of(t, mt, nb, width);
      const bool g0 = 64 * part < width, g1 = 64 * part + 32 < width;   // this thread's code groups
      // the row's slot and scale (and, for the sign pass, its code words and the parts of
      // ||r||^2) are loaded before the accumulation, so their latency hides under it
      const int64_t r = mt * kGenTile + row;              // row within the chunk
      int64_t slot = r < A.n ? (A.slots ? A.slots[A.row0 + r] : A.row0 + r) : 0;
      const bool live = r < A.n && slot >= 0 && slot < A.cap;   // (the prep kernel reported a bad slot)
      if (!live) slot = 0;
      const RowInfo ri = live ? A.info[r] : RowInfo{0.f, 0.f};
      uint32_t* rec = reinterpret_cast<uint32_t*>(A.codes + slot * (int64_t)A.code_bytes);
      uint32_t old[2][P];
      float rn2_all = 0.f;
      if constexpr (SIGN) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int grp = (nb * kGenNb) / 32 + 2 * part + h;
#pragma unroll
          for (int p = 0; p < P; ++p) old[h][p] = (live && (h ? g1 : g0)) ? rec[grp * P + p] : 0u;
        }
        if (live && nb == 0 && part == 0)
          for (int j = 0; j < 4 * A.NB; ++j) rn2_all += A.rn2[r * A.NB * 4 + j];
      }
      float acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = 0.f;
      for (int a = 0; a < KA; ++a, ++q) {
        const int b = (int)(q & 1);
        if (!wait(acc_full + b, (uint32_t)((q >> 1) & 1))) { fail(404); ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < 2 ? g0 : g1) {
            uint32_t raw[16];
            tmem_ld16(lane_base + (uint32_t)(b * kGenNb + 64 * part + 16 * c), raw);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[16 * c + i] += __uint_as_float(raw[i]);
          }
        }
        tc_fence_before();
        mbar_arrive(acc_empty + b);
      }
      if (!ok) break;
      float rn2 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!(h ? g1 : g0)) continue;
        const int grp = (nb * kGenNb) / 32 + 2 * part + h;   // code group of these 32 coordinates
        const int i0 = 32 * grp;
        uint32_t w[P];
#pragma unroll
        for (int p = 0; p < P; ++p) w[p] = 0u;
        if constexpr (!SIGN) {
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool in = i0 + e < A.d;
            const float y = acc[32 * h + e] * ri.inv;
            const bool pos = y > 0.f;
            const float av = fabsf(y);
            int m = 0;
#pragma unroll
            for (int j = 0; j < LEVELS / 2 - 1; ++j) m += av > A.pos_t[j] ? 1 : 0;
            uint32_t code = KB == 1 ? (pos ? 0u : 1u) : ((pos ? 0u : 1u) << (KB - 1)) | (uint32_t)m;
            float rr = y - (pos ? A.mag[m] : -A.mag[m]);
            if (!in) code = 0u;
            if (!in || ri.nrm == 0.f) rr = 0.f;
#pragma unroll
            for (int bit = 0; bit < KB; ++bit) {
              const int qb = code_bit_pos(P, e, bit);
              w[qb >> 5] |= ((code >> bit) & 1u) << (qb & 31);
            }
            if constexpr (PROD) {
              rn2 = fmaf(rr, rr, rn2);
              const float sr = rr * kGenRScale;
              const __half hh = __float2half_rn(sr);
              const __half ll = __float2half_rn(sr - __half2float(hh));
              if (e & 1) {
                hi[e >> 1] |= (uint32_t)__half_as_ushort(hh) << 16;
                lo[e >> 1] |= (uint32_t)__half_as_ushort(ll) << 16;
              } else {
                hi[e >> 1] = __half_as_ushort(hh);
                lo[e >> 1] = __half_as_ushort(ll);
              }
            }
          }
          if (live) {
#pragma unroll
            for (int p = 0; p < P; ++p) rec[grp * P + p] = w[p];
            if constexpr (PROD) {
              uint4* dh = reinterpret_cast<uint4*>(A.R + r * A.K + i0);
              uint4* dl = reinterpret_cast<uint4*>(A.R + (A.lo_off + r) * A.K + i0);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                dh[u] = make_uint4(hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3]);
                dl[u] = make_uint4(lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3]);
              }
            }
          }
        } else {
          // QJL signs [z >= 0] of the coordinates < d into the top code bit
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool bit = (i0 + e < A.d) && (acc[32 * h + e] >= 0.f);
            const int qb = code_bit_pos(P, e, P - 1);
            w[qb >> 5] |= (bit ? 1u : 0u) << (qb & 31);
          }
          if (live)
#pragma unroll
            for (int p = 0; p < P; ++p) rec[grp * P + p] = old[h][p] | w[p];
        }
      }
      if constexpr (!SIGN) {
        // partial ||r||^2 of this thread's columns: 4 parts per N block
        if (PROD && live) A.rn2[(r * A.NB + nb) * 4 + part] = rn2;
      } else {
        if (live && nb == 0 && part == 0)
          A.rnorm[slot] = ri.nrm > 0.f ? __half_as_ushort(__float2half_rn(sqrtf(rn2_all))) : (uint16_t)0;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int P, int KB, bool PROD, bool SIGN>
int launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int sms, cudaStream_t st) {
  constexpr int STAGE = 2 * kGenTile * 128 + 2 * kGenNb * 128;
  const int smem_bytes = kGenStages * STAGE + 256 + 1024;
  auto kern = quantize_gemm_kernel<P, KB, PROD, SIGN>;
  cudaError_t e = ensure_smem_attrs<quantize_gemm_kernel<P, KB, PROD, SIGN>>(smem_bytes, false);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(quantize_gemm)");
  const int64_t units = (a.rows / kGenTile) * a.NB;
  const int grid = (int)std::min<int64_t>(units, sms);
  (void)STAGE;
  kern<<<grid, kGenThreads, smem_bytes, st>>>(ta, tb, a);
  count_launch();
  return check_launch("quantize_gemm_kernel");
}

template <bool SIGN>
int launch_gemm(int P, int KB, bool prod, const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int sms,
                cudaStream_t st) {
#define TQ_GEN(PP, KK, PR) \
  if (P == PP && KB == KK && prod == PR) return launch_gemm_t<PP, KK, PR, SIGN>(ta, tb, a, sms, st);
  if constexpr (!SIGN) {
    TQ_GEN(1, 1, false) TQ_GEN(2, 2, false) TQ_GEN(3, 3, false) TQ_GEN(4, 4, false)
  }
  TQ_GEN(2, 1, true) TQ_GEN(3, 2, true) TQ_GEN(4, 3, true) TQ_GEN(5, 4, true)
#undef TQ_GEN
  return fail(TQ_ERR_INTERNAL, "quantize: no projection kernel for this code layout");
}

}  // namespace

size_t quantize_gen_workspace(const tq_ctx* ctx, int64_t n) { return gen_layout(ctx, n).total; }

// Quantize n rows of x through the workspace (any d, fp32 / fp16 / bf16 input).
int launch_quantize_gen(const tq_ctx* ctx, const void* x, int x_dtype, int64_t n, int64_t ld, const int32_t* cols,
                        const tq_packed* dst, const int64_t* slots, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!ctx->Pi16 || (ctx->mode == TQ_MODE_PROD && !ctx->M16))
    return fail(TQ_ERR_INTERNAL, "context has no tensor-core projection operands");
  const GenLayout L = gen_layout(ctx, n);
  if (!ws || ws_bytes < L.total) return fail(TQ_ERR_WORKSPACE, "quantize: workspace too small");
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(TQ_ERR_UNSUPPORTED, "quantize: workspace must be 256-byte aligned");
  char* base = static_cast<char*>(ws);
  __half* X = reinterpret_cast<__half*>(base + L.off_x);
  __half* R = reinterpret_cast<__half*>(base + L.off_r);
  RowInfo* info = reinterpret_cast<RowInfo*>(base + L.off_info);
  float* rn2 = reinterpret_cast<float*>(base + L.off_rn2);
  const bool prod = ctx->mode == TQ_MODE_PROD;
  const int P = ctx->lay.planes, KB = ctx->lay.k;
  CUtensorMap tx, tr, tpi, tm;
  if (!make_map(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)L.rows, L.K, (uint64_t)L.K * 2, kGenTile) ||
      !make_map(&tpi, ctx->Pi16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)L.N, L.K, (uint64_t)L.K * 2,
                (uint32_t)std::min(kGenNb, L.N)))
    return fail(TQ_ERR_INTERNAL, "quantize: tensor maps");
  if (prod && (!make_map(&tr, R, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)L.rows, L.K, (uint64_t)L.K * 2, kGenTile) ||
               !make_map(&tm, ctx->M16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2 * (uint64_t)L.N, L.K, (uint64_t)L.K * 2,
                         (uint32_t)std::min(kGenNb, L.N))))
    return fail(TQ_ERR_INTERNAL, "quantize: tensor maps");
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, ctx->device);
  GemmArgs g{};
  g.K = L.K;
  g.N = L.N;
  g.NB = L.NB;
  g.d = ctx->lay.d;
  g.code_bytes = ctx->lay.code_bytes;
  g.slots = slots;
  g.codes = dst->codes;
  g.rnorm = dst->rnorm;
  g.info = info;
  g.R = R;
  g.rn2 = rn2;
  g.err = ctx->dev_err;
  g.cap = dst->cap;
  g.wait_ns = pipeline_wait_ns();
  const int lev = ctx->cb.K;
  for (int j = 0; j < 8; ++j) {
    g.pos_t[j] = (j + 1 < lev / 2) ? ctx->cb.t[lev / 2 - 1 + j + 1] : INFINITY;
    g.mag[j] = (j < lev / 2) ? ctx->cb.c[lev / 2 + j] : 0.f;
  }
  if (lev == 2) g.mag[0] = ctx->cb.c[1];
  g.lo_off = L.rows;
  g.box_b = std::min(kGenNb, L.N);
  for (int64_t row0 = 0; row0 < n; row0 += L.rows) {
    const int64_t cn = std::min<int64_t>(L.rows, n - row0);
    const int64_t rows = (cn + kGenTile - 1) / kGenTile * kGenTile;
    PrepArgs p{};
    p.x = x;
    p.cols = cols;
    p.ld = ld;
    p.n = cn;
    p.row0 = row0;
    p.d = ctx->lay.d;
    p.K = L.K;
    p.slots = slots;
    p.norm = dst->norm;
    p.X = X;
    p.R = prod ? R : nullptr;
    p.N = L.N;
    p.rows = rows;
    p.lo_off = L.rows;
    p.cap = dst->cap;
    p.info = info;
    p.err = ctx->dev_err;
    const int pgrid = (int)((rows + 7) / 8);
    if (x_dtype == TQ_DTYPE_F32) quantize_prep_kernel<float><<<pgrid, 256, 0, st>>>(p);
    else if (x_dtype == TQ_DTYPE_F16) quantize_prep_kernel<__half><<<pgrid, 256, 0, st>>>(p);
    else quantize_prep_kernel<__nv_bfloat16><<<pgrid, 256, 0, st>>>(p);
    count_launch();
    int r = check_launch("quantize_prep_kernel");
    if (r != TQ_OK) return r;
    g.n = cn;
    g.rows = rows;
    g.row0 = row0;
    r = launch_gemm<false>(P, KB, prod, tx, tpi, g, sms, st);
    if (r != TQ_OK) return r;
    if (prod) {
      r = launch_gemm<true>(P, KB, prod, tr, tm, g, sms, st);
      if (r != TQ_OK) return r;
    }
  }
  return TQ_OK;
}

}  // namespace tq
