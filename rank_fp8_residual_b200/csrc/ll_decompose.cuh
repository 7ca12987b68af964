// Residual quantisation of the LiteLinear decomposition (sm_100a)
//
// After the SVD of a dense weight W ~= A B (LiteLinear README, "Usage":
// LiteLinear.from_dense, an SVD-based decomposition; A = U_r S_r, B = V_r^T
// as the MoDeGPT compressor keeps them), the layer stores the residual
// R = W - A B as e4m3fn codes with a multiplier ("Features": Q_fp8 and
// Q_scale_inv):
//
//   R[n, k] = W[n, k] - sum_j A[n, j] B[j, k]      binary64, j in order
//   scale   = max |R| / 448, rounded to binary32   (per row or per tensor)
//   Q[n, k] = e4m3fn(binary32(R[n, k] / scale))    nearest, ties to even
//
// Every rounding step is fixed (explicit round-to-nearest binary64
// intrinsics, never contracted into fused multiply-adds), so each code is
// decided in exactly the precision stated above.  A set-time operation on
// CUDA cores: one block per weight row, the row of R kept in shared memory
// between its maximum and its codes.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"

namespace llk {

constexpr int kRqThreads = 256;

__device__ __forceinline__ double bf16_bits_to_double(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

// Row n of R into shared memory (Rs, K doubles); returns the block-wide
// max |R[n, :]| to every thread.
__device__ double rq_row(const uint16_t* __restrict__ W, const uint16_t* __restrict__ A,
                         const uint16_t* __restrict__ B, int n, int K, int r, double* Rs, double* As,
                         double* red) {
  for (int j = threadIdx.x; j < r; j += blockDim.x) As[j] = bf16_bits_to_double(A[static_cast<size_t>(n) * r + j]);
  __syncthreads();
  double amax = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    double acc = 0.0;
    for (int j = 0; j < r; ++j)
      acc = __dadd_rn(acc, __dmul_rn(As[j], bf16_bits_to_double(B[static_cast<size_t>(j) * K + k])));
    const double v = __dsub_rn(bf16_bits_to_double(W[static_cast<size_t>(n) * K + k]), acc);
    Rs[k] = v;
    amax = fmax(amax, fabs(v));
  }
  // block maximum
  for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  double m = 0.0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) m = fmax(m, red[i]);
  __syncthreads();  // Rs, As and red are reused by the caller / next row
  return m;
}

__device__ __forceinline__ void rq_codes(const double* Rs, int K, float s, uint8_t* __restrict__ Qrow) {
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    uint8_t c = 0;
    if (s != 0.f) {
      const float u = __double2float_rn(__ddiv_rn(Rs[k], static_cast<double>(s)));
      c = static_cast<uint8_t>(f32x2_to_e4m3x2(u, 0.f) & 0xFFu);
    }
    Qrow[k] = c;
  }
}

// Per-row scales: one block per row (grid-stride), codes and scale[n].
// Per-tensor scale, first pass: rowmax[n] only.
__global__ void __launch_bounds__(kRqThreads) ll_residual_rows_kernel(const uint16_t* __restrict__ W,
                                                                      const uint16_t* __restrict__ A,
                                                                      const uint16_t* __restrict__ B, int N, int K,
                                                                      int r, uint8_t* __restrict__ Q,
                                                                      float* __restrict__ scale,
                                                                      double* __restrict__ rowmax) {
  extern __shared__ double rq_smem[];
  double* red = rq_smem;        // 32
  double* As = red + 32;        // r
  double* Rs = As + r;          // K
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const double m = rq_row(W, A, B, n, K, r, Rs, As, red);
    if (rowmax != nullptr) {
      if (threadIdx.x == 0) rowmax[n] = m;
      continue;
    }
    const float s = __double2float_rn(__ddiv_rn(m, 448.0));
    if (threadIdx.x == 0) scale[n] = s;
    rq_codes(Rs, K, s, Q + static_cast<size_t>(n) * K);
    __syncthreads();
  }
}

// Per-tensor scale, second pass: the tensor maximum from rowmax, then R
// again and the codes.
__global__ void __launch_bounds__(kRqThreads) ll_residual_tensor_kernel(const uint16_t* __restrict__ W,
                                                                        const uint16_t* __restrict__ A,
                                                                        const uint16_t* __restrict__ B, int N,
                                                                        int K, int r, uint8_t* __restrict__ Q,
                                                                        float* __restrict__ scale,
                                                                        const double* __restrict__ rowmax) {
  extern __shared__ double rq_smem[];
  double* red = rq_smem;
  double* As = red + 32;
  double* Rs = As + r;
  double g = 0.0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) g = fmax(g, rowmax[i]);
  for (int o = 16; o > 0; o >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = g;
  __syncthreads();
  double m = 0.0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) m = fmax(m, red[i]);
  __syncthreads();
  const float s = __double2float_rn(__ddiv_rn(m, 448.0));
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = s;
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    rq_row(W, A, B, n, K, r, Rs, As, red);
    rq_codes(Rs, K, s, Q + static_cast<size_t>(n) * K);
    __syncthreads();
  }
}

__host__ __device__ constexpr size_t rq_smem_bytes(int K, int r) {
  return sizeof(double) * (32 + static_cast<size_t>(r) + static_cast<size_t>(K));
}

}  // namespace llk
