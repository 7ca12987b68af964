// CUDA-core GEMV path (sm_100a) of the LiteLinear forward for M <= 4 tokens
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// At a few tokens the forward is a matrix-vector product bound by reading
// Q (N*K bytes), A (2*N*r) and B (2*r*K) from HBM once; the tensor core's
// 128-row MMA would be idle but for 1/32 of its N side.  Here every weight
// element is used by M <= 4 fused multiply-adds on CUDA cores, with warp
// reductions:
//
//   ll_gemv_t_kernel   t[m, j] = sum_k x[m, k] B[j, k]          (fp32)
//   ll_gemv_kernel     acc_Q[m, n] = sum_k x[m, k] dec(Q[n, k]),
//                      acc_LR[m, n] = sum_j t[m, j] A[n, j],
//                      y[m, n] = bf16(scale[n] acc_Q + (acc_LR + bias[n]))
//
// Products are exact in fp32 (an e4m3fn value has 4 significant bits, a
// bf16 value 8) and are summed in fp32: per lane in K order, then across
// the lanes of a warp in a fixed butterfly order.
//
// Streaming.  A warp owns kGvRows output features and walks their rows in
// chunks of 512 bytes (512 codes of Q, or 256 columns of A): each lane
// copies its own 16 bytes of each row with cp.async into a warp-private
// ring of kGvStages chunks and later reads back exactly those bytes, so a
// wait_group suffices and no barrier is needed.  Sixteen warps per CTA, one
// CTA per SM: up to 128 KB of loads in flight per SM.  x sits in shared
// memory for the CTA's lifetime; t is read from global memory (L2) after
// the t kernel, the programmatic primary, has completed.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

constexpr int kGvMaxM = 4;
constexpr int kGvWarps = 16;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kGvRows = 4;    // output features per warp task
constexpr int kGvStages = 4;  // chunks in flight per warp
constexpr int kGvChunk = 512;  // bytes of one row per chunk
constexpr int kGvRingBytes = kGvWarps * kGvStages * kGvRows * kGvChunk;  // 128 KB

__host__ __device__ constexpr size_t gv_smem_bytes(int M, int K) {
  return static_cast<size_t>(kGvRingBytes) + static_cast<size_t>(M) * K * 2 + 128;
}

struct GemvParams {
  const uint16_t* x;     // [M, K] bf16
  const uint8_t* q;      // [N, K] e4m3fn codes
  const uint16_t* a;     // [N, r_pad] bf16
  const float* t;        // [M, r_pad] fp32, written by ll_gemv_t_kernel
  const float* scale;    // [N]
  const uint16_t* bias;  // [N] or nullptr
  uint16_t* y;           // [M, N]
  int M, N, K, r_pad;
  int t_from_primary;    // 1: t is written by the preceding kernel
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %2, 0;\n\t"
      "@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}" ::"r"(smem_u32(smem)),
      "l"(gmem), "r"(static_cast<int>(pred))
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kN>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kN) : "memory");
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// x rows into shared memory, 16 bytes per thread per step.
__device__ __forceinline__ void gv_load_x(const uint16_t* __restrict__ x, uint16_t* xs, int M, int K) {
  const int n16 = M * K / 8;
  for (int i = threadIdx.x; i < n16; i += blockDim.x)
    reinterpret_cast<uint4*>(xs)[i] = __ldg(reinterpret_cast<const uint4*>(x) + i);
  __syncthreads();
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// t = x B^T: one warp per row j of B (grid-stride), lanes over K.
template <int kM>
__global__ void __launch_bounds__(kGvThreads) ll_gemv_t_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ B,
                                                               float* __restrict__ t, int K, int r_pad) {
  constexpr int M = kM;
  pdl_launch_dependents();  // the main kernel's residual stream does not need t
  extern __shared__ __align__(16) uint8_t gv_smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(gv_smem);
  gv_load_x(x, xs, M, K);
  const int lane = threadIdx.x & 31;
  const int wg = blockIdx.x * kGvWarps + (threadIdx.x >> 5), nw = gridDim.x * kGvWarps;
  for (int j = wg; j < r_pad; j += nw) {
    float acc[kM];
#pragma unroll
    for (int m = 0; m < kM; ++m) acc[m] = 0.f;
    // eight loads of the row in flight per lane, then their products
    for (int kb = lane * 8; kb < K; kb += 256 * 8) {
      uint4 bv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int k0 = kb + 256 * u;
        bv[u] = k0 < K ? __ldg(reinterpret_cast<const uint4*>(B + static_cast<size_t>(j) * K + k0)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int k0 = kb + 256 * u;
        if (k0 < K) {
          float b[8];
          bf16x8_to_f32(bv[u], b);
#pragma unroll
          for (int m = 0; m < kM; ++m) {
            float xv[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(xs + m * K + k0), xv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[m] = fmaf(xv[i], b[i], acc[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kM; ++m) {
      const float s = warp_sum(acc[m]);
      if (lane == 0) t[m * r_pad + j] = s;
    }
  }
}

template <int kM, int kAct>
__global__ void __launch_bounds__(kGvThreads, 1) ll_gemv_kernel(const __grid_constant__ GemvParams p) {
  extern __shared__ __align__(16) uint8_t gv_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = gv_smem + warp * (kGvStages * kGvRows * kGvChunk);  // this warp's chunks
  uint16_t* xs = reinterpret_cast<uint16_t*>(gv_smem + kGvRingBytes);
  gv_load_x(p.x, xs, kM, p.K);

  constexpr int M = kM;
  const int K = p.K;
  const int nQ = (K + kGvChunk - 1) / kGvChunk;               // residual chunks per row
  const int nA = (p.r_pad * 2 + kGvChunk - 1) / kGvChunk;      // low-rank chunks per row
  const int nC = nQ + nA;
  const int tasks = (p.N + kGvRows - 1) / kGvRows;
  bool waited = false;
  // Task t goes to CTA t % grid, so the tasks spread evenly over the SMs.
  for (int task = blockIdx.x + gridDim.x * warp; task < tasks; task += gridDim.x * kGvWarps) {
    const int n0 = task * kGvRows;
    // This lane's 16 bytes of row i in chunk c.
    auto issue = [&](int c) {
      uint8_t* st = ring + (c % kGvStages) * (kGvRows * kGvChunk) + lane * 16;
      if (c < nC) {
        const bool qc = c < nQ;
        const int col = (qc ? c : c - nQ) * kGvChunk + lane * 16;  // byte within the row
        const int row_bytes = qc ? K : 2 * p.r_pad;
#pragma unroll
        for (int i = 0; i < kGvRows; ++i) {
          const int n = n0 + i;
          const bool ok = n < p.N && col < row_bytes;
          const uint8_t* src = qc ? p.q + static_cast<size_t>(n) * K + col
                                  : reinterpret_cast<const uint8_t*>(p.a) + static_cast<size_t>(n) * p.r_pad * 2 + col;
          cp_async16(st + i * kGvChunk, ok ? src : p.q, ok);
        }
      }
      cp_async_commit();  // an empty group past the last chunk keeps the count uniform
    };
#pragma unroll
    for (int c = 0; c < kGvStages - 1; ++c) issue(c);
    float aq[kGvRows][kM], al[kGvRows][kM];
#pragma unroll
    for (int i = 0; i < kGvRows; ++i)
#pragma unroll
      for (int m = 0; m < kM; ++m) aq[i][m] = al[i][m] = 0.f;
    for (int c = 0; c < nC; ++c) {
      issue(c + kGvStages - 1);
      cp_async_wait<kGvStages - 1>();  // chunk c (this lane's own bytes) has landed
      const uint8_t* st = ring + (c % kGvStages) * (kGvRows * kGvChunk) + lane * 16;
      if (c < nQ) {
        const int k0 = c * kGvChunk + lane * 16;
        if (k0 < K) {
          uint4 qv[kGvRows];
#pragma unroll
          for (int i = 0; i < kGvRows; ++i) qv[i] = *reinterpret_cast<const uint4*>(st + i * kGvChunk);
          // x[m, k0 + 8 g .. + 7] against codes 8 g .. 8 g + 7 of each row
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            float xv[kM][8];
#pragma unroll
            for (int m = 0; m < kM; ++m) bf16x8_to_f32(*reinterpret_cast<const uint4*>(xs + m * K + k0 + 8 * g), xv[m]);
#pragma unroll
            for (int i = 0; i < kGvRows; ++i) {
              const uint32_t w0 = g ? qv[i].z : qv[i].x, w1 = g ? qv[i].w : qv[i].y;
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float2 d = e4m3x2_to_f32x2(static_cast<uint16_t>((h < 2 ? w0 : w1) >> (16 * (h & 1))));
#pragma unroll
                for (int m = 0; m < kM; ++m) {
                  aq[i][m] = fmaf(xv[m][2 * h], d.x, aq[i][m]);
                  aq[i][m] = fmaf(xv[m][2 * h + 1], d.y, aq[i][m]);
                }
              }
            }
          }
        }
      } else {
        const int j0 = (c - nQ) * (kGvChunk / 2) + lane * 8;  // column of A and t
        if (j0 < p.r_pad) {
          if (!waited && p.t_from_primary) {
            pdl_wait_primary();
            waited = true;
          }
          float tv[kM][8];
#pragma unroll
          for (int m = 0; m < kM; ++m) {
              const float4 t0 = __ldcg(reinterpret_cast<const float4*>(p.t + m * p.r_pad + j0));
              const float4 t1 = __ldcg(reinterpret_cast<const float4*>(p.t + m * p.r_pad + j0 + 4));
              tv[m][0] = t0.x; tv[m][1] = t0.y; tv[m][2] = t0.z; tv[m][3] = t0.w;
              tv[m][4] = t1.x; tv[m][5] = t1.y; tv[m][6] = t1.z; tv[m][7] = t1.w;
            }
#pragma unroll
          for (int i = 0; i < kGvRows; ++i) {
            float av[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(st + i * kGvChunk), av);
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
              for (int m = 0; m < kM; ++m) al[i][m] = fmaf(tv[m][e], av[e], al[i][m]);
          }
        }
      }
    }
    cp_async_wait<0>();
    // Sums across the warp; lane i * 4 + m holds (row i, token m).
#pragma unroll
    for (int i = 0; i < kGvRows; ++i)
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        const float sq = warp_sum(aq[i][m]);
        const float sl = warp_sum(al[i][m]);
        const int n = n0 + i;
        if (lane == i * kGvMaxM + m && n < p.N) {
          const float b = p.bias != nullptr ? bf16_bits_to_float(p.bias[n]) : 0.f;
          p.y[static_cast<size_t>(m) * p.N + n] = to_bf16_bits(epi_act<kAct>(fmaf(__ldg(p.scale + n), sq, sl + b)));
        }
      }
  }
}

}  // namespace llk
