// Top-k search over a packed database on the 5th-generation tensor cores (tcgen05).
//
// turboquant.net "向量搜索中的应用" / admirer.cn vector-search paragraph: every database
// vector is stored quantized and a query ranks the database by the unbiased estimator
//   score(q, k) = ||k|| ( <Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, 2 s - 1> ),
// top-k by score, ties to the lower id.  For a tile of 128 queries and a chunk of 256
// database vectors that is ONE dense product over K = 2 Kh (Kh = 64 ceil(d/64)):
//
//   D [128 x 256] = Q [128 x K] * B [256 x K]^T,   score = ||k|| D
//   Q row  = ( Pi q | sqrt(pi/2)/m S q )                 fp16, built once per query
//   B row  = ( c[idx] | +-||r|| )                        fp16, decoded per chunk from the codes
//
// with the two halves interleaved per 64-coordinate atom (centroid atom, then sign atom of
// the same coordinates) so one read of the code words feeds both.  ||r|| is an fp16 value,
// so +-||r|| is exact; the centroids and the query carry fp16 rounding (2^-11 relative),
// which moves a unit-vector score by ~1e-5.
//
// Roles (576 threads per CTA, one CTA per SM for a fixed query tile): warp 0 stages the
// query atoms by TMA (and, for 4-bit codes, the chunk's code words into a ring); warp 1
// owns TMEM (two 256-column accumulators) and issues the MMAs; warps 2-9 decode database
// atoms (thread = database row: code words -> fp16 by byte-permute table lookups ->
// 128-byte-swizzled shared memory) and stage the chunk's norms; warps 10-17 are the
// epilogue (thread = query x half of the chunk's columns when k <= 32, else query x all
// of them on warps 10-13: scores from TMEM, a running top-k list in shared memory with
// the k-th score as threshold).
// At the end every list is written as candidates; the search merge kernel takes the top-k
// of each query over the lists of its query tile.  Every wait is bounded; a timeout
// records an error code in the context's error word and the CTA winds down.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_ops.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

using namespace sm100;
using mmaops::prmt;

constexpr int kSqM = 128;                 // queries per tile
constexpr int kSqN = 256;                 // database vectors per chunk
constexpr int kSqStages = 2;
constexpr int kSqCStages = 4;             // ring of code tiles (4-bit codes): 256 rows x 32 bytes each
constexpr int kSqCStage = kSqN * 32;
constexpr int kSqDecWarps = 8;
constexpr int kSqEpiWarps = 8;            // two per TMEM lane quarter: each takes half of a chunk's columns
constexpr int kSqHalfK = 32;               // the two halves keep separate lists when k <= this
constexpr int kSqThreads = 64 + 32 * (kSqDecWarps + kSqEpiWarps);
constexpr int kSqMaxK = 64;
constexpr uint64_t kSqWaitNs = 2000000000ull;
constexpr int kSqStageA = kSqM * 128;     // 16 KB
constexpr int kSqStageB = kSqN * 128;     // 32 KB
constexpr int kSqStage = kSqStageA + kSqStageB;

struct SqArgs {
  const uint8_t* codes;
  const uint16_t* norm;
  const uint16_t* rnorm;
  int64_t N;                 // database vectors
  int nq, d, Kh, code_bytes, k;
  int cpq;                   // CTAs per query tile
  int halves;                // epilogue lists per query and CTA (2 when k <= kSqHalfK, else 1)
  int64_t nchunks;
  float* cand_s;             // [nq][cpq * halves * k]
  int64_t* cand_i;
  uint32_t ctab_lo[2], ctab_hi[2];   // 3-bit (neg, magnitude) code -> signed centroid fp16 bytes (P = 4)
  uint32_t ctab[32];                 // P-bit code -> signed centroid fp16 (other P)
  uint64_t wait_ns;                  // limit of the pipeline waits
  int* err;
};

template <int P>
__global__ void __launch_bounds__(kSqThreads, 1) search_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_c,
                                                                  const SqArgs A) {
  // 4-bit codes: the code words of each 64-coordinate block of the chunk (256 rows x 32
  // bytes) are staged by TMA into a ring a few blocks ahead of the decoders; other widths
  // are read by the decoders straight from global memory
  constexpr bool RING = P == 4;
  extern __shared__ uint8_t sq_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sq_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cring = smem + kSqStages * kSqStage;                                  // [cstages][256][32]
  float* list_s = reinterpret_cast<float*>(cring + (RING ? kSqCStages * kSqCStage : 0));   // [k][128]
  int32_t* list_i = reinterpret_cast<int32_t*>(list_s + kSqMaxK * kSqM);          // [k][128]
  float* s_norm = reinterpret_cast<float*>(list_i + kSqMaxK * kSqM);              // [2][256]
  uint32_t* s_ctab = reinterpret_cast<uint32_t*>(s_norm + 2 * kSqN);              // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_ctab + 32);
  uint64_t* full_a = bars;                          // [stages] TMA
  uint64_t* full_b = bars + kSqStages;              // [stages] decoders
  uint64_t* empty = bars + 2 * kSqStages;           // [stages] MMA commit
  uint64_t* acc_full = bars + 3 * kSqStages;        // [2]
  uint64_t* acc_empty = acc_full + 2;               // [2]
  uint64_t* nrm_full = acc_empty + 2;               // [2] chunk norms staged
  uint64_t* nrm_empty = nrm_full + 2;               // [2] chunk norms consumed
  uint64_t* drain = nrm_empty + 2;
  uint64_t* cfull = drain + 1;                      // [cstages] code tile landed
  uint64_t* cempty = cfull + kSqCStages;            // [cstages] code tile decoded
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + kSqCStages);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x / A.cpq, cslot = blockIdx.x % A.cpq;
  const int nloc = (int)((A.nchunks - cslot + A.cpq - 1) / A.cpq);
  const int KA = 2 * A.Kh / 64;                     // atoms per chunk (centroid + sign)
  constexpr int kDecThreads = 32 * kSqDecWarps;
  const int kEpiThreads = 32 * (A.halves == 2 ? kSqEpiWarps : kSqEpiWarps / 2);   // active epilogue threads

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSqStages; ++s) {
      mbar_init(full_a + s, 1);
      mbar_init(full_b + s, kDecThreads);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, kEpiThreads);
      mbar_init(nrm_full + b, kDecThreads);
      mbar_init(nrm_empty + b, kEpiThreads);
    }
    mbar_init(drain, 1);
    for (int c = 0; c < kSqCStages; ++c) {
      mbar_init(cfull + c, 1);
      mbar_init(cempty + c, kDecThreads);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 32) s_ctab[threadIdx.x] = A.ctab[threadIdx.x];
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

  if (warp == 0) {
    // --------------------------------------------------------------- query atoms (TMA)
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      int pending[kSqStages];
      for (int s = 0; s < kSqStages; ++s) pending[s] = -1;
      int64_t q = 0;
      bool ok = true;
      for (int t = 0; ok && t < nloc; ++t)
        for (int a = 0; a < KA; ++a, ++q) {
          const int s = (int)(q % kSqStages);
          const uint32_t ph = (uint32_t)((q / kSqStages) & 1);
          if (!wait(empty + s, ph ^ 1)) { fail(501); ok = false; break; }
          mbar_arrive_expect_tx(full_a + s, kSqStageA);
          tma_load_2d(smem + s * kSqStage, &tm_q, 64 * a, qt * kSqM, full_a + s);
          pending[s] = (int)ph;
        }
      for (int s = 0; s < kSqStages; ++s)
        if (pending[s] >= 0) mbar_wait(full_a + s, (uint32_t)pending[s], nullptr, kSqWaitNs);
    } else if (RING && lane == 1) {
      // code tiles of every 64-coordinate block of every chunk, kSqCStages ahead
      prefetch_tensormap(&tm_c);
      int pending[kSqCStages];
      for (int c = 0; c < kSqCStages; ++c) pending[c] = -1;
      int64_t cq = 0;
      bool ok = true;
      for (int t = 0; ok && t < nloc; ++t) {
        const int64_t chunk = cslot + (int64_t)t * A.cpq;
        for (int pr = 0; pr < KA / 2; ++pr, ++cq) {
          const int c = (int)(cq % kSqCStages);
          const uint32_t ph = (uint32_t)((cq / kSqCStages) & 1);
          if (!wait(cempty + c, ph ^ 1)) { fail(507); ok = false; break; }
          mbar_arrive_expect_tx(cfull + c, kSqCStage);
          tma_load_2d(cring + c * kSqCStage, &tm_c, 32 * pr, (int)(chunk * kSqN), cfull + c);
          pending[c] = (int)ph;
        }
      }
      for (int c = 0; c < kSqCStages; ++c)
        if (pending[c] >= 0) mbar_wait(cfull + c, (uint32_t)pending[c], nullptr, kSqWaitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kSqM, kSqN, 0);
      int64_t q = 0;
      bool ok = true;
      for (int t = 0; ok && t < nloc; ++t) {
        const int b = t & 1;
        if (!wait(acc_empty + b, (uint32_t)(((t >> 1) & 1) ^ 1))) { fail(502); break; }
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(b * kSqN);
        for (int a = 0; a < KA; ++a, ++q) {
          const int s = (int)(q % kSqStages);
          const uint32_t ph = (uint32_t)((q / kSqStages) & 1);
          if (!wait(full_a + s, ph) || !wait(full_b + s, ph)) { fail(503); ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * kSqStage);
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(dcol, desc_sw128(base + kk * 32), desc_sw128(base + kSqStageA + kk * 32), idesc,
                   (a | kk) ? 1u : 0u);
          mma_commit(empty + s);
        }
        if (!ok) break;
        mma_commit(acc_full + b);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, kSqWaitNs);
    }
  } else if (warp < 2 + kSqDecWarps) {
    // --------------------------------------------------------------- database decoders
    const int row = threadIdx.x - 64;               // database row of the chunk
    const int rsw = row & 7;
    const uint32_t tl0 = A.ctab_lo[0], tl1 = A.ctab_lo[1], th0 = A.ctab_hi[0], th1 = A.ctab_hi[1];
    const int NG = (A.d + 31) / 32;                 // code groups
    int64_t q = 0;
    bool ok = true;
    // the row's norm and residual norm of chunk t + 1 load while chunk t is decoded
    auto norms_of = [&](int tt, uint16_t& nv, uint16_t& rv) {
      const int64_t idn = (cslot + (int64_t)tt * A.cpq) * kSqN + row;
      nv = 0;
      rv = 0;
      if (tt < nloc && idn < A.N) {
        nv = __ldg(A.norm + idn);
        rv = __ldg(A.rnorm + idn);
      }
    };
    uint16_t nxt_n, nxt_r;
    norms_of(0, nxt_n, nxt_r);
    for (int t = 0; ok && t < nloc; ++t) {
      const int64_t chunk = cslot + (int64_t)t * A.cpq;
      const int64_t id = chunk * kSqN + row;
      const bool live = id < A.N;
      const uint8_t* rec = A.codes + (live ? id : 0) * (int64_t)A.code_bytes;
      const uint16_t cur_n = nxt_n, cur_r = nxt_r;   // zero for a row past the database
      norms_of(t + 1, nxt_n, nxt_r);
      // the chunk's norms for the epilogue
      const int nb = t & 1;
      if (!wait(nrm_empty + nb, (uint32_t)(((t >> 1) & 1) ^ 1))) { fail(504); ok = false; break; }
      s_norm[nb * kSqN + row] = __half2float(__ushort_as_half(cur_n));
      mbar_arrive(nrm_full + nb);
      const uint32_t rbits = (uint32_t)cur_r & 0x7FFFu;
      const uint32_t rr = rbits | (rbits << 16);
      uint32_t w[2][P];                             // code words of the atom's two groups
      for (int a = 0; a < KA; ++a, ++q) {
        const int s = (int)(q % kSqStages);
        const uint32_t ph = (uint32_t)((q / kSqStages) & 1);
        const int ca = a >> 1;                      // 64-coordinate block
        const bool sign_atom = a & 1;
        const int64_t cq = (int64_t)t * (KA / 2) + ca;   // code tile of this block
        if (RING && !sign_atom) {
          const int c = (int)(cq % kSqCStages);
          if (!wait(cfull + c, (uint32_t)((cq / kSqCStages) & 1))) { fail(508); ok = false; break; }
          const uint4* src = reinterpret_cast<const uint4*>(cring + c * kSqCStage + row * 32);
          const uint4 v0 = src[0], v1 = src[1];
          w[0][0] = v0.x; w[0][1] = v0.y; w[0][2] = v0.z; w[0][3] = v0.w;
          w[1][0 % P] = v1.x; w[1][1 % P] = v1.y; w[1][2 % P] = v1.z; w[1][3 % P] = v1.w;
          mbar_arrive(cempty + c);                  // the words are in registers
        } else if (!RING && !sign_atom) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int g = 2 * ca + h;
            if (live && g < NG) {
              if constexpr (P == 4) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(rec + 16 * g));
                w[h][0] = v.x; w[h][1] = v.y; w[h][2] = v.z; w[h][3] = v.w;
              } else {
#pragma unroll
                for (int p = 0; p < P; ++p) w[h][p] = __ldg(reinterpret_cast<const uint32_t*>(rec) + g * P + p);
              }
            } else {
#pragma unroll
              for (int p = 0; p < P; ++p) w[h][p] = 0u;
            }
          }
        }
        if (!wait(empty + s, ph ^ 1)) { fail(505); ok = false; break; }
        uint8_t* dst = smem + s * kSqStage + kSqStageA + (row >> 3) * 1024 + rsw * 128;
        // No range checks: coordinates >= d and rows past the database decode from zero
        // words, the record's padding bytes or another row's codes, all to finite fp16
        // values; those coordinates meet zero query entries (the query operand is zero past
        // d) and those rows never enter a list (id >= N).
        {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {            // 8-coordinate slice u of group g: one 16-byte chunk
              uint32_t o[4];
              if (!sign_atom) {
                if constexpr (P == 4) {
                  const uint32_t sel = w[h][u] & 0x77777777u;
#pragma unroll
                  for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t sl = hh ? sel >> 16 : sel;
                    const uint32_t lb = prmt(tl0, tl1, sl), hb = prmt(th0, th1, sl);
                    o[2 * hh] = prmt(lb, hb, 0x5140u);
                    o[2 * hh + 1] = prmt(lb, hb, 0x7362u);
                  }
                } else {
#pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    const uint32_t va = s_ctab[group_code(w[h], P, 8 * u + e)];
                    const uint32_t vb = s_ctab[group_code(w[h], P, 8 * u + e + 1)];
                    o[e / 2] = (va & 0xFFFFu) | (vb << 16);
                  }
                }
              } else if constexpr (P == 4) {
                // +-||r||: the fp16 sign bit set where the QJL sign bit is 0.  The sign bits of
                // coordinates 0-3 are the byte msbs of the word, those of 4-7 after a shift by 4.
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  const uint32_t nm = ~(hh ? w[h][u] << 4 : w[h][u]);
                  o[2 * hh] = (prmt(nm, 0u, 0x1404u) & 0x80008000u) | rr;
                  o[2 * hh + 1] = (prmt(nm, 0u, 0x3424u) & 0x80008000u) | rr;
                }
              } else {
                // +-||r||: the fp16 sign bit set where the QJL sign bit is 0
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  const uint32_t sa = (w[h][code_bit_pos(P, 8 * u + e, P - 1) >> 5] >> (code_bit_pos(P, 8 * u + e, P - 1) & 31)) & 1u;
                  const uint32_t sb =
                      (w[h][code_bit_pos(P, 8 * u + e + 1, P - 1) >> 5] >> (code_bit_pos(P, 8 * u + e + 1, P - 1) & 31)) & 1u;
                  o[e / 2] = rr | ((sa ^ 1u) << 15) | ((sb ^ 1u) << 31);
                }
              }
              const int chunk16 = h * 4 + u;          // 16-byte chunk of the 128-byte row
              *reinterpret_cast<uint4*>(dst + ((chunk16 ^ rsw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(full_b + s);
      }
    }
  } else {
    // ----------------------------------------------------------------------- epilogue
    // warp e: TMEM lane quarter warp & 3 (query rows), column half e >> 2 of each chunk; with
    // one half (k > kSqHalfK) the first four warps take all 256 columns and the rest idle
    const int e = warp - 2 - kSqDecWarps;
    const int wq = warp & 3;
    const int half = e >> 2;
    const bool active = A.halves == 2 || half == 0;
    const int col0 = A.halves == 2 ? half * (kSqN / 2) : 0;
    const int ncol = A.halves == 2 ? kSqN / 2 : kSqN;
    const int qr = wq * 32 + lane;                  // query row of the tile (TMEM lane)
    const int li = A.halves == 2 ? half * kSqM + qr : qr;   // this thread's list
    const int ls = A.halves * kSqM;                 // list stride between entries
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const int k = A.k;
    if (active) {
      for (int j = 0; j < k; ++j) {
        list_s[j * ls + li] = -INFINITY;
        list_i[j * ls + li] = INT32_MAX;
      }
      float tau = -INFINITY;
      for (int t = 0; t < nloc; ++t) {
        const int b = t & 1;
        const int64_t chunk = cslot + (int64_t)t * A.cpq;
        if (!wait(acc_full + b, (uint32_t)((t >> 1) & 1)) || !wait(nrm_full + b, (uint32_t)((t >> 1) & 1))) {
          fail(506);
          break;
        }
        tc_fence_after();
        for (int g = 0; g < ncol / 32; ++g) {
          uint32_t raw[32];
          tmem_ld32(lane_base + (uint32_t)(b * kSqN + col0 + 32 * g), raw);
          tmem_ld_wait();
          if (g == ncol / 32 - 1) {
            tc_fence_before();
            mbar_arrive(acc_empty + b);
          }
          // the 32 scores first, then one test against the list's threshold: most groups
          // of 32 hold no candidate once the list has filled
          float sv[32];
          float smax = -INFINITY;
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            sv[e2] = __uint_as_float(raw[e2]) * s_norm[b * kSqN + col0 + 32 * g + e2];
            smax = fmaxf(smax, sv[e2]);
          }
          if (!(smax > tau)) continue;
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            const int c = col0 + 32 * g + e2;
            const float sc = sv[e2];
            const int64_t id = chunk * kSqN + c;
            if (sc > tau && id < A.N) {
              // insert (ids rise within a list, so a later equal score stays behind)
              int pos = k - 1;
              while (pos > 0 && list_s[(pos - 1) * ls + li] < sc) {
                list_s[pos * ls + li] = list_s[(pos - 1) * ls + li];
                list_i[pos * ls + li] = list_i[(pos - 1) * ls + li];
                --pos;
              }
              list_s[pos * ls + li] = sc;
              list_i[pos * ls + li] = (int32_t)id;
              tau = list_s[(k - 1) * ls + li];
            }
          }
        }
        mbar_arrive(nrm_empty + b);
      }
      const int qg = qt * kSqM + qr;
      if (qg < A.nq) {
        const int64_t per_q = (int64_t)A.cpq * A.halves * k;
        const int64_t o = (int64_t)qg * per_q + ((int64_t)cslot * A.halves + (A.halves == 2 ? half : 0)) * k;
        for (int j = 0; j < k; ++j) {
          const int32_t id = list_i[j * ls + li];
          A.cand_s[o + j] = list_s[j * ls + li];
          A.cand_i[o + j] = id == INT32_MAX ? INT64_MAX : (int64_t)id;
        }
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

// Query operand: row q = per 64-coordinate block a, (Pi q)[64a .. 64a+64) then
// sqrt(pi/2)/m (S q)[64a .. 64a+64), fp16, zero beyond d; rows >= nq are zero.  A tiled fp32
// product [nq x d] x [d x d] per part: CTA = 64 queries x 64 outputs, K in steps of 16
// through shared memory, thread = 4 queries x 4 outputs.
__global__ void __launch_bounds__(256) search_query_kernel(const float* __restrict__ q, int64_t nq, int d, int Kh,
                                                           const float* __restrict__ PiT, const float* __restrict__ ST,
                                                           float coef, __half* __restrict__ out) {
  __shared__ float Qs[16][68];                       // [k][query]
  __shared__ float Ms[16][68];                       // [k][output]
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  const int o0 = blockIdx.y * 64, part = blockIdx.z;
  const float* M = part == 0 ? PiT : ST;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < d; k0 += 16) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int qq = e >> 4, kk = e & 15;
      Qs[kk][qq] = (r0 + qq < nq && k0 + kk < d) ? __ldg(q + (r0 + qq) * d + k0 + kk) : 0.f;
      const int kr = e >> 6, oo = e & 63;
      Ms[kr][oo] = (k0 + kr < d && o0 + oo < d) ? __ldg(M + (size_t)(k0 + kr) * d + o0 + oo) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = Qs[kk][ty * 4 + i];
        bv[i] = Ms[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float sc = part == 0 ? 1.f : coef;
  const int64_t K = 2 * (int64_t)Kh;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = r0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tx * 4 + j;
      if (o < Kh) out[row * K + (int64_t)(o / 64) * 128 + part * 64 + (o % 64)] = __float2half_rn(acc[i][j] * sc);
    }
  }
}

// The same product for d a multiple of 8 (16-byte rows): CTA = 128 queries x 128 outputs of
// one part, thread = 8 queries x 8 outputs (two 4 x 4 blocks 64 apart, so every shared-memory
// read is one conflict-free 16-byte load), K in steps of 8 with the next step's global loads
// in flight during the current step's 512 FMAs.  Every output sums its d terms in the same
// order as the kernel above, so the two give identical operands.
constexpr int kQgTile = 128;
__global__ void __launch_bounds__(256) search_query_gemm_kernel(const float* __restrict__ q, int64_t nq, int d, int Kh,
                                                                const float* __restrict__ PiT,
                                                                const float* __restrict__ ST, float coef,
                                                                __half* __restrict__ out) {
  __shared__ __align__(16) float As[2][8][kQgTile + 4];   // [buffer][k][query]
  __shared__ __align__(16) float Bs[2][8][kQgTile];       // [buffer][k][output]
  const int64_t r0 = (int64_t)blockIdx.x * kQgTile;
  const int o0 = blockIdx.y * kQgTile, part = blockIdx.z;
  const float* M = part == 0 ? PiT : ST;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  // loader roles: A row t/2, k half t%2 (one 16-byte load); B k row t/32, outputs 4 (t%32)
  const int ar = t >> 1, ak = 4 * (t & 1), bk = t >> 5, bo = 4 * (t & 31);
  const bool a_ok = r0 + ar < nq, b_ok = o0 + bo < d;
  const float* qa = q + (a_ok ? (r0 + ar) * d : 0) + ak;
  const float* mb = M + (b_ok ? o0 + bo : 0) + (size_t)bk * d;
  float4 ra = make_float4(0.f, 0.f, 0.f, 0.f), rb = ra;
  auto fetch = [&](int k0) {
    if (a_ok) ra = __ldg(reinterpret_cast<const float4*>(qa + k0));
    if (b_ok) rb = __ldg(reinterpret_cast<const float4*>(mb + (size_t)k0 * d));
  };
  auto put = [&](int buf) {
    As[buf][ak + 0][ar] = ra.x;
    As[buf][ak + 1][ar] = ra.y;
    As[buf][ak + 2][ar] = ra.z;
    As[buf][ak + 3][ar] = ra.w;
    *reinterpret_cast<float4*>(&Bs[buf][bk][bo]) = rb;
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int nk = d / 8;
  fetch(0);
  put(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) fetch(8 * (kt + 1));
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][64 + 4 * tx]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kt + 1 < nk) put(cur ^ 1);
    __syncthreads();
  }
  const float sc = part == 0 ? 1.f : coef;
  const int64_t K = 2 * (int64_t)Kh;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = r0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
#pragma unroll
    for (int jb = 0; jb < 2; ++jb) {
      const int o = o0 + 64 * jb + 4 * tx;   // four outputs inside one 64-coordinate block
      if (o < Kh) {
        const __half2 lo = __floats2half2_rn(acc[i][4 * jb] * sc, acc[i][4 * jb + 1] * sc);
        const __half2 hi = __floats2half2_rn(acc[i][4 * jb + 2] * sc, acc[i][4 * jb + 3] * sc);
        uint2 v;
        v.x = *reinterpret_cast<const uint32_t*>(&lo);
        v.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + row * K + (int64_t)(o / 64) * 128 + part * 64 + (o % 64)) = v;
      }
    }
  }
}

struct SqWs {
  size_t qop, cs, ci, total;
  int cpq, qtiles, Kh;
  int64_t nq_pad;
};

SqWs sq_ws(const tq_ctx* ctx, int64_t nq, int k, int sms) {
  SqWs w{};
  w.Kh = 64 * ((ctx->lay.d + 63) / 64);
  w.qtiles = (int)((nq + kSqM - 1) / kSqM);
  w.nq_pad = (int64_t)w.qtiles * kSqM;
  w.cpq = std::max(1, sms / std::max(1, w.qtiles));
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.qop = 0;
  w.cs = up((size_t)w.nq_pad * 2 * w.Kh * sizeof(__half));
  const int halves = k <= kSqHalfK ? 2 : 1;
  w.ci = w.cs + up((size_t)nq * w.cpq * halves * k * sizeof(float));
  w.total = w.ci + up((size_t)nq * w.cpq * halves * k * sizeof(int64_t));
  return w;
}

int device_sms(int dev) {
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}

template <int P>
int launch_sq_t(const CUtensorMap& tmq, const CUtensorMap& tmc, const SqArgs& a, int grid, cudaStream_t st) {
  const int smem = kSqStages * kSqStage + (P == 4 ? kSqCStages * kSqCStage : 0) + 2 * kSqMaxK * kSqM * 4 +
                   2 * kSqN * 4 + 32 * 4 + 256 + 1024;
  auto kern = search_tc_kernel<P>;
  cudaError_t e = ensure_smem_attrs<search_tc_kernel<P>>(smem, false);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(search_tc)");
  kern<<<grid, kSqThreads, smem, st>>>(tmq, tmc, a);
  count_launch();
  return check_launch("search_tc_kernel");
}

}  // namespace

size_t search_tc_workspace(const tq_ctx* ctx, int64_t nq, int64_t N, int k) {
  (void)N;
  return sq_ws(ctx, nq, k, device_sms(ctx->device)).total;
}

// Any prod-mode database, k <= 64.
int launch_search_tc(const tq_ctx* ctx, const float* q, int64_t nq, const tq_packed* db, int64_t N, int k,
                     float* scores, int64_t* ids, void* ws, cudaStream_t st) {
  if (ctx->mode != TQ_MODE_PROD) return fail(TQ_ERR_INVALID_ARG, "search needs a prod-mode context");
  if (k < 1 || k > kSqMaxK) return fail(TQ_ERR_UNSUPPORTED, "search: k must be in [1, 64]");
  if (nq == 0) return TQ_OK;
  const int sms = device_sms(ctx->device);
  const SqWs W = sq_ws(ctx, nq, k, sms);
  char* base = static_cast<char*>(ws);
  __half* qop = reinterpret_cast<__half*>(base + W.qop);
  float* cs = reinterpret_cast<float*>(base + W.cs);
  int64_t* ci = reinterpret_cast<int64_t*>(base + W.ci);
  const int d = ctx->lay.d;
  // the query operand
  if (d % 8 == 0 && (reinterpret_cast<uintptr_t>(q) & 15) == 0) {
    const dim3 grid((unsigned)(W.nq_pad / kQgTile), (unsigned)((W.Kh + kQgTile - 1) / kQgTile), 2);
    search_query_gemm_kernel<<<grid, 256, 0, st>>>(q, nq, d, W.Kh, ctx->PiT, ctx->ST, ctx->sqrt_pi_over_2_over_m,
                                                   qop);
    count_launch();
    int r = check_launch("search_query_gemm_kernel");
    if (r != TQ_OK) return r;
  } else {
    const dim3 grid((unsigned)(W.nq_pad / 64), (unsigned)((W.Kh + 63) / 64), 2);
    search_query_kernel<<<grid, 256, 0, st>>>(q, nq, d, W.Kh, ctx->PiT, ctx->ST, ctx->sqrt_pi_over_2_over_m, qop);
    count_launch();
    int r = check_launch("search_query_kernel");
    if (r != TQ_OK) return r;
  }
  CUtensorMap tmq;
  if (!make_map(&tmq, qop, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)W.nq_pad, 2 * (uint64_t)W.Kh,
                2 * (uint64_t)W.Kh * 2, kSqM))
    return fail(TQ_ERR_INTERNAL, "search: tensor map of the query operand");
  CUtensorMap tmc = tmq;
  if (ctx->lay.planes == 4 &&
      !make_map_plain(&tmc, db->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)N, (uint64_t)ctx->lay.code_bytes,
                      (uint64_t)ctx->lay.code_bytes, 32, kSqN))
    return fail(TQ_ERR_INTERNAL, "search: tensor map of the database codes");
  SqArgs a{};
  a.codes = db->codes;
  a.norm = db->norm;
  a.rnorm = db->rnorm;
  a.N = N;
  a.nq = (int)nq;
  a.d = d;
  a.Kh = W.Kh;
  a.code_bytes = ctx->lay.code_bytes;
  a.k = k;
  a.cpq = W.cpq;
  a.halves = k <= kSqHalfK ? 2 : 1;
  a.nchunks = (N + kSqN - 1) / kSqN;
  a.cand_s = cs;
  a.cand_i = ci;
  a.err = ctx->dev_err;
  a.wait_ns = pipeline_wait_ns();
  const int kb = ctx->lay.k, P = ctx->lay.planes;
  auto signed_centroid = [&](uint32_t code) -> __half {
    const int idx = code_index(code & ((1u << kb) - 1u), kb);
    return __float2half_rn((float)ctx->host.centroids[idx]);
  };
  for (int code = 0; code < 32; ++code)
    a.ctab[code] = code < (1 << P) ? (uint32_t)__half_as_ushort(signed_centroid((uint32_t)code)) : 0u;
  if (P == 4) {
    uint8_t lo[8], hi[8];
    for (int c = 0; c < 8; ++c) {
      const uint16_t v = __half_as_ushort(signed_centroid((uint32_t)c));
      lo[c] = (uint8_t)(v & 0xFF);
      hi[c] = (uint8_t)(v >> 8);
    }
    for (int r = 0; r < 2; ++r) {
      a.ctab_lo[r] = lo[4 * r] | (lo[4 * r + 1] << 8) | (lo[4 * r + 2] << 16) | ((uint32_t)lo[4 * r + 3] << 24);
      a.ctab_hi[r] = hi[4 * r] | (hi[4 * r + 1] << 8) | (hi[4 * r + 2] << 16) | ((uint32_t)hi[4 * r + 3] << 24);
    }
  }
  const int grid = W.qtiles * W.cpq;
  int r;
  switch (P) {
    case 2: r = launch_sq_t<2>(tmq, tmc, a, grid, st); break;
    case 3: r = launch_sq_t<3>(tmq, tmc, a, grid, st); break;
    case 4: r = launch_sq_t<4>(tmq, tmc, a, grid, st); break;
    case 5: r = launch_sq_t<5>(tmq, tmc, a, grid, st); break;
    default: return fail(TQ_ERR_INTERNAL, "search: code layout");
  }
  if (r != TQ_OK) return r;
  return launch_search_merge(cs, ci, nq, (int64_t)W.cpq * a.halves * k, k, scores, ids, st);
}

}  // namespace tq
