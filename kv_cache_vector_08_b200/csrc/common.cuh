// Internal definitions shared by the libtq CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstdint>
#include <string>

#include <cuda.h>

#include "../../include/tq.h"
#include "params.h"

namespace tq {

constexpr int kMaxLevels = 16;  // 2^k for k <= 4

// Codebook and layout constants passed to kernels by value.
struct Codebook {
  float c[kMaxLevels];      // centroids, ascending
  float t[kMaxLevels];      // boundaries (K-1 used); t[K-1..] = +inf
  float cc[kMaxLevels];     // centroid of each sign-magnitude index code (see index_code)
  int K;                    // 2^k
};

struct Layout {
  int d, d_pad, k, planes, code_bytes;   // planes = P code bits per coordinate
};

// Sign-magnitude code of a k-bit codebook index (the packed-code convention): bit k-1 is
// the negative-half flag [idx < K/2], the low bits the magnitude rank counted from the
// centre of the (odd-symmetric) codebook; for k = 1 the code is the flag alone.
__host__ __device__ inline uint32_t index_code(int idx, int k) {
  const int half = 1 << (k - 1);
  if (k == 1) return idx == 0 ? 1u : 0u;
  const bool neg = idx < half;
  return ((neg ? 1u : 0u) << (k - 1)) | (uint32_t)(neg ? half - 1 - idx : idx - half);
}
__host__ __device__ inline int code_index(uint32_t code, int k) {
  const int half = 1 << (k - 1);
  if (k == 1) return (code & 1u) ? 0 : 1;
  const int m = (int)(code & (uint32_t)(half - 1));
  return ((code >> (k - 1)) & 1u) ? half - 1 - m : half + m;
}

// Position of code bit b of coordinate e (0..31) of a 32-coordinate group with P-bit
// codes, as 32 * word + bit (the record layout stated with the packed format).
__host__ __device__ constexpr int code_bit_pos(int P, int e, int b) {
  return P == 1 ? (8 * ((e & 7) & 3) + 7 - (2 * (e >> 3) + ((e & 7) >> 2)))
       : (b == P - 1 && P != 4) ? 32 * (P - 1) + (8 * ((e & 7) & 3) + 7 - (2 * (e >> 3) + ((e & 7) >> 2)))
       : P == 2 ? 4 * (e & 7) + (e >> 3)
       : P == 3 ? 32 * ((e >> 3) & 1) + 4 * (e & 7) + 2 * (e >> 4) + b
       : b == 3 ? 32 * (e >> 3) + ((((e & 7) >> 2) == 0) ? 8 * (e & 3) + 7 : 8 * (e & 3) + 3)
       : 32 * (e >> 3) + 4 * (e & 7) + b;
}

// P-bit code of coordinate e of a group whose P words are in w.
__device__ __forceinline__ uint32_t group_code(const uint32_t* w, int P, int e) {
  uint32_t c = 0;
  for (int b = 0; b < P; ++b) {
    const int q = code_bit_pos(P, e, b);
    c |= ((w[q >> 5] >> (q & 31)) & 1u) << b;
  }
  return c;
}

}  // namespace tq

struct tq_ctx {
  tq::HostParams host;
  int device = 0;
  tq::Layout lay{};
  tq::Codebook cb{};
  int m = 0, mode = 0, bits = 0;
  float sqrt_pi_over_2_over_m = 0.f;  // QJL unbiasing constant sqrt(pi/2)/m
  float s_rowmax = 0.f;               // max_j ||S_j||: bounds |(S q)_j| by s_rowmax * ||q||
  // device float32 copies (row-major): Pi for the decode merge's inverse rotation, the
  // transposes for the query projections (coalesced column access)
  float* Pi = nullptr;    // [d][d]    y = Pi x
  float* PiT = nullptr;   // [d][d]    Pi^T
  float* ST = nullptr;    // [d][m]    S^T
  // tensor-core operands (d in {64, 128}): Pi as three bf16 splits [3][d][d] and
  // 16 * M as two fp16 splits [2][d][d], row-major
  void* Pi_split = nullptr;
  void* M_split = nullptr;
  // dequantize operand (d <= 128): 16 Pi^T as fp16 hi / lo, [2][N][d_pad] with
  // N = 16 ceil(d/16), row n holding 16 Pi[k][n] over k (zero padded)
  void* PiT_f16 = nullptr;
  // QJL-augmented dequantize operand (prod mode, d <= 128): 16 sqrt(pi/2)/m S^T as fp16
  // hi / lo, same layout (row n holding 16 kappa S[k][n] over k)
  void* ST_f16 = nullptr;
  // projection operands of the workspace quantize path (any d): 16 Pi and 16 M as fp16 hi /
  // lo, [2][d_pad][K] with K = 64 ceil(d/64), row n holding 16 Pi[n][k] (16 M[n][k])
  void* Pi16 = nullptr;
  void* M16 = nullptr;
  int* dev_err = nullptr;  // device error word written by kernels that detect a stuck pipeline
};

namespace tq {

void set_error(const std::string& msg);
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

// Kernel attributes persist on a device: the dynamic shared-memory limit is raised only when
// a launch needs more than any earlier launch of this kernel on the current device, and the
// maximum carveout is requested once, instead of two driver calls before every launch.
// (Like every attribute, they do not survive a cudaDeviceReset.)
constexpr int kAttrDevices = 64;
template <auto Kern>
inline cudaError_t ensure_smem_attrs(int dyn_bytes, bool max_carveout) {
  static int dyn_set[kAttrDevices];
  static bool carve_set[kAttrDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kAttrDevices) {
    cudaGetLastError();
    dev = -1;
  }
  if (dev < 0 || dyn_bytes > dyn_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_bytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0) dyn_set[dev] = dyn_bytes;
  }
  if (max_carveout && (dev < 0 || !carve_set[dev])) {
    const cudaError_t e =
        cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    if (dev >= 0) carve_set[dev] = true;
  }
  return cudaSuccess;
}
void count_launch(uint64_t n = 1);

// Limit of the pipeline waits of the dequantize, search and workspace-quantize kernels
// (2 s unless a test changed it with tq_debug_set_wait_limit).
uint64_t pipeline_wait_ns();
// Test hook: the dequantize kernel's MMA issuer first waits on a barrier that nothing
// arrives on (tq_debug_inject_stall), so that wait runs out after pipeline_wait_ns().
bool debug_stall();
// Device allocation of tq_init (a test can make the n-th one fail, see tq_debug_fail_alloc).
cudaError_t dev_alloc(void** p, size_t bytes);

// Kernel-side error codes written to the context's error word (first one wins).
enum DeviceError : int {
  kErrSlotRange = 901,   // a slot index outside [0, cap) was passed in a device slot array: the row is skipped
  kErrPermRange = 902,   // a channel permutation / column map entry outside [0, D): the element is skipped
};

// 2-D row-major tensor map [rows][cols] of 16-bit elements with box {64 columns, box_rows
// rows} and 128-byte swizzle (the canonical K-major operand layout of tcgen05.mma).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
              uint64_t row_stride_bytes, uint32_t box_rows);
// 2-D row-major tensor map with box {box_cols, box_rows} and no swizzle.
bool make_map_plain(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows);

// Returns TQ_OK if the last launch succeeded, else records the error.
int check_launch(const char* what);

inline int div_up(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace tq
