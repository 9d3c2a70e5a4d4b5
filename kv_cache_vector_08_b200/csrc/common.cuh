// Internal definitions shared by the libtq CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstdint>
#include <string>

#include "../../include/tq.h"
#include "params.h"

namespace tq {

constexpr int kMaxLevels = 16;  // 2^k for k <= 4

// Codebook and layout constants passed to kernels by value.
struct Codebook {
  float c[kMaxLevels];      // centroids, ascending
  float t[kMaxLevels];      // boundaries (K-1 used); t[K-1..] = +inf
  int K;                    // 2^k
};

struct Layout {
  int d, d_pad, k, planes, code_bytes;
  int quarter;              // d_pad / 4 coordinate positions per quarter
  int chunk;                // d_pad / 32 bytes per plane inside a quarter
  int qbytes;               // planes * chunk bytes per quarter
};

// Byte offset, inside one vector's record, of the byte holding plane p of positions
// [i, i+8) (i a multiple of 8).
__host__ __device__ inline int plane_byte(const Layout& L, int p, int i) {
  int q = i / L.quarter;
  return q * L.qbytes + p * L.chunk + (i - q * L.quarter) / 8;
}

}  // namespace tq

struct tq_ctx {
  tq::HostParams host;
  int device = 0;
  tq::Layout lay{};
  tq::Codebook cb{};
  int m = 0, mode = 0, bits = 0;
  float sqrt_pi_over_2_over_m = 0.f;  // QJL unbiasing constant sqrt(pi/2)/m
  // device float32 copies (row-major)
  float* Pi = nullptr;    // [d][d]    y = Pi x
  float* PiT = nullptr;   // [d][d]    Pi^T (coalesced column access)
  float* S = nullptr;     // [m][d]
  float* ST = nullptr;    // [d][m]
  float* MT = nullptr;    // [d][m]    (S Pi^T)^T
  // tensor-core operands (d in {64, 128}): Pi as three bf16 splits [3][d][d] and
  // 16 * M as two fp16 splits [2][d][d], row-major
  void* Pi_split = nullptr;
  void* M_split = nullptr;
  int* dev_err = nullptr;  // device error word written by kernels that detect a stuck pipeline
};

namespace tq {

void set_error(const std::string& msg);
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);
void count_launch(uint64_t n = 1);

// Returns TQ_OK if the last launch succeeded, else records the error.
int check_launch(const char* what);

inline int div_up(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace tq
