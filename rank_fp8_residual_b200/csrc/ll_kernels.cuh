// CUDA kernels (sm_100a) of the LiteLinear forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// with x [M,K] bf16, B [r,K] bf16, A [N,r] bf16, Q [N,K] e4m3fn codes,
// scale [N] fp32, bias [N] bf16, y [M,N] bf16 (README "Features" and "Usage"
// give the dtypes; SVDLinearLayer on the tt_compressor page gives the
// factor shapes).
//
// Kernel chain for one forward (all on the caller's stream):
//   1. ll_lrdown_kernel   t = x B^T with tcgen05, fp32 accumulate in TMEM,
//                         written as a bf16 pair (t_hi = bf16(t),
//                         t_lo = bf16(t - t_hi)).  With several K splits
//                         the splits of a tile form one cluster and add
//                         their partial sums in split order over
//                         distributed shared memory.
//   2. ll_main_kernel     persistent fused GEMM.  Tile = 128 output
//                         features x up to 128 tokens.  Q (e4m3fn) is the
//                         MMA A operand: converter warps widen it exactly to
//                         bf16 and write it into tensor memory; x is the MMA
//                         B operand, brought to shared memory by TMA.  The
//                         low-rank part accumulates A * (t_hi + t_lo)^T into
//                         a second TMEM accumulator.  The epilogue applies
//                         y = scale[n]*acc_Q + acc_LR + bias[n] in fp32,
//                         rounds once to bf16 and writes with TMA stores.
//                         It is launched with programmatic dependent launch
//                         and waits for kernel 1 only before its first
//                         read of t, so its x*Q^T main loop overlaps them.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace llk {

enum : int {
  kErrTimeoutProducer = 0x101,
  kErrTimeoutMma = 0x102,
  kErrTimeoutConvert = 0x103,
  kErrTimeoutEpilogue = 0x104,
  kErrTimeoutDrain = 0x105,
};

constexpr int kBK = 64;  // K elements per pipeline step (128 bytes of bf16)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait used while draining after an error: ignores the status
// word, gives up after the timeout.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, const Watch& w) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = clock_cycles();
  while (!mbar_try_wait(a, parity)) {
    if (clock_cycles() - t0 > 2ull * w.timeout_ns) {
      atomicCAS(w.status, 0, kErrTimeoutDrain);
      return;
    }
  }
}

// =====================================================================
// Kernel 1: t = x B^T
// =====================================================================
struct LrDownParams {
  CUtensorMap tm_x;  // bf16 [M, K]      box {64, 128}, 128B swizzle
  CUtensorMap tm_b;  // bf16 [r_pad, K]  box {64, rc},  128B swizzle
  uint16_t* t_hi;    // [M, r_pad] bf16 bits
  uint16_t* t_lo;    // [M, r_pad]
  int M, K, r_pad;
  int rc;            // box height of B = column block of t per CTA (<= 256)
  int tmem_cols;     // power of two >= rc
  int ksplit;        // number of K splits (gridDim.z; one cluster along z when > 1)
  int kb_per_split;  // 64-wide K steps per split
  const int* e_tok;  // [M] token exponents: t is written divided by 2^e_tok[m]; nullptr: unscaled
  int wait_prior;    // 1: e_tok comes from the kernel before (programmatic dependent launch): wait for
                     // it before the epilogue, and let this kernel's dependents launch only then
  Watch watch;
};

__device__ __forceinline__ float exp2_int(int e) { return __int_as_float((127 + e) << 23); }

// Ring depth: as many stages as fit in 192 KB (4 to 8): t's reads of x come
// from HBM, so the more bytes in flight the closer to its bandwidth.
constexpr int kLrMaxStages = 8;
constexpr int kLrRingBytes = 192 * 1024;
constexpr int kLrThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr int kLrMaxSplit = 8;   // K splits per tile = CTAs per cluster (portable limit)

__host__ __device__ constexpr int lr_stage_bytes(int rc) { return 128 * kBK * 2 + rc * kBK * 2; }
__host__ __device__ constexpr int lr_stages(int rc) {
  return kLrRingBytes / lr_stage_bytes(rc) < kLrMaxStages ? kLrRingBytes / lr_stage_bytes(rc) : kLrMaxStages;
}
__host__ constexpr int lr_smem_bytes(int rc) { return lr_stages(rc) * lr_stage_bytes(rc) + 1024 + 256; }

// Position of float4 column c4 of partial-sum row `row` in shared memory:
// rows of rc fp32, the eight float4 of each 32-column block permuted by
// row so that a warp's 32 rows store without bank conflicts.
__device__ __forceinline__ uint32_t lr_part_off(int row, int c4, int rc) {
  return static_cast<uint32_t>(row * rc * 4 + (((c4 & ~7) | ((c4 ^ row) & 7)) << 4));
}

__global__ void __launch_bounds__(kLrThreads, 1) ll_lrdown_kernel(const __grid_constant__ LrDownParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int stage_bytes = lr_stage_bytes(p.rc);
  const int n_stages = lr_stages(p.rc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + n_stages * stage_bytes);
  uint64_t* empty = full + n_stages;
  uint64_t* acc_full = empty + n_stages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int j0 = blockIdx.y * p.rc;
  const int wcols = min(p.rc, p.r_pad - j0);  // columns of t this CTA owns (multiple of 32)
  const int kz = blockIdx.z;                  // K split = rank in the cluster
  const int nK = (p.K + kBK - 1) / kBK;
  const int kb_begin = kz * p.kb_per_split;
  const int kb_end = min(nK, kb_begin + p.kb_per_split);
  const int ncols = p.tmem_cols;

  // Producer state (thread 0): the first lap of the ring is issued before
  // the TMEM allocation and the block barrier.
  int ps = 0, issued = 0;
  uint32_t pph = 0;
  if (threadIdx.x == 0) {
    if (!p.wait_prior) pdl_launch_dependents();
    for (int s = 0; s < n_stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    for (int kb = kb_begin; kb < kb_end && issued < n_stages; ++kb, ++issued) {
      uint8_t* st = smem + issued * stage_bytes;
      mbar_arrive_expect_tx(&full[issued], stage_bytes);
      tma_load_2d(st, &p.tm_x, &full[issued], kb * kBK, m0);
      tma_load_2d(st + 128 * kBK * 2, &p.tm_b, &full[issued], kb * kBK, j0);
    }
    ps = issued % n_stages;
    pph = issued == n_stages ? 1u : 0u;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = kb_begin + issued; kb < kb_end; ++kb) {
        if (!mbar_wait(&empty[ps], pph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
        uint8_t* st = smem + ps * stage_bytes;
        mbar_arrive_expect_tx(&full[ps], stage_bytes);
        tma_load_2d(st, &p.tm_x, &full[ps], kb * kBK, m0);
        tma_load_2d(st + 128 * kBK * 2, &p.tm_b, &full[ps], kb * kBK, j0);
        ++issued;
        if (++ps == n_stages) { ps = 0; pph ^= 1; }
      }
      if (!ok) {
        // Let every load already issued land before the CTA can exit.
        for (int i = max(0, issued - n_stages); i < issued; ++i)
          mbar_wait_drain(&full[i % n_stages], (i / n_stages) & 1, p.watch);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, wcols);
      int s = 0;
      uint32_t ph = 0;
      bool first = true;
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(&full[s], ph, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * stage_bytes);
        const uint64_t ad = sdesc_kmajor_sw128(st);
        const uint64_t bd = sdesc_kmajor_sw128(st + 128 * kBK * 2);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          mma_ss(tbase, ad + 2 * kk, bd + 2 * kk, idesc, first ? 0u : 1u);
          first = false;
        }
        tc_commit(&empty[s]);
        if (++s == n_stages) { s = 0; ph ^= 1; }
      }
      tc_commit(acc_full);
      // No MMA may still run when TMEM is released below.
      tc_commit(drain);
      mbar_wait_drain(drain, 0, p.watch);
    }
  } else {
    // Epilogue: TMEM lane = token row.  One split: the bf16 pair straight to
    // global memory.  Several: this split's fp32 partial into this CTA's
    // shared memory (the ring is idle once every MMA is done).
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int m = m0 + row;
    if (p.wait_prior) {
      // The token exponents are written by the kernel before this one.
      pdl_wait_primary();
      if (warp == 2 && lane == 0) pdl_launch_dependents();
    }
    if (__all_sync(0xffffffffu, mbar_wait(acc_full, 0, p.watch, kErrTimeoutEpilogue))) {
      tc_fence_after();
      const bool empty_range = kb_end <= kb_begin;
      for (int c = 0; c < wcols; c += 32) {
        uint32_t v[32];
        tmem_ld32_wait(tbase + ((32u * q) << 16) + c, v);
        if (empty_range) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (p.ksplit > 1) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4*>(smem + lr_part_off(row, c / 4 + i, p.rc)) =
                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                            __uint_as_float(v[4 * i + 3]));
        } else if (m < p.M) {
          // exact: a power-of-two scaling of a value far from both ends of the range
          const float mult = p.e_tok != nullptr ? exp2_int(-p.e_tok[m]) : 1.f;
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = __uint_as_float(v[2 * i]) * mult;
            const float b = __uint_as_float(v[2 * i + 1]) * mult;
            const uint16_t ha = to_bf16_bits(a), hb = to_bf16_bits(b);
            hi[i] = static_cast<uint32_t>(ha) | (static_cast<uint32_t>(hb) << 16);
            lo[i] = pack_bf16x2(a - bf16_bits_to_float(ha), b - bf16_bits_to_float(hb));
          }
          uint4* dh = reinterpret_cast<uint4*>(p.t_hi + static_cast<size_t>(m) * p.r_pad + j0 + c);
          uint4* dl = reinterpret_cast<uint4*>(p.t_lo + static_cast<size_t>(m) * p.r_pad + j0 + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dh[i] = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
            dl[i] = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, ncols);
  }
  if (p.ksplit == 1) return;
  if (p.wait_prior) pdl_wait_primary();  // the reduction below reads the token exponents

  // Split K: the CTAs of a cluster hold the partials of one tile; after the
  // cluster barrier, CTA kz sums rows [kz * rpc, (kz + 1) * rpc) of every
  // split's partial over distributed shared memory, in split order, and
  // writes the bf16 pair.  Every CTA reaches both cluster barriers, also
  // after a timeout.
  cluster_sync();
  const int rows = min(128, p.M - m0);
  const int rpc = (rows + p.ksplit - 1) / p.ksplit;
  const int r0 = kz * rpc;
  const int r1 = min(rows, r0 + rpc);
  const int q4 = wcols / 4;
  const int total = max(0, r1 - r0) * q4;
  const uint32_t sbase = smem_u32(smem);
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int row = r0 + i / q4;
    const int c4 = i % q4;
    const uint32_t off = sbase + lr_part_off(row, c4, p.rc);
    float4 v[kLrMaxSplit];
#pragma unroll
    for (int z = 0; z < kLrMaxSplit; ++z)
      if (z < p.ksplit) v[z] = ld_shared_cluster_f4(mapa_shared(off, static_cast<uint32_t>(z)));
    float4 acc = v[0];
#pragma unroll
    for (int z = 1; z < kLrMaxSplit; ++z)
      if (z < p.ksplit) {
        acc.x += v[z].x;
        acc.y += v[z].y;
        acc.z += v[z].z;
        acc.w += v[z].w;
      }
    if (p.e_tok != nullptr) {
      const float mult = exp2_int(-p.e_tok[m0 + row]);
      acc.x *= mult;
      acc.y *= mult;
      acc.z *= mult;
      acc.w *= mult;
    }
    const uint16_t h0 = to_bf16_bits(acc.x), h1 = to_bf16_bits(acc.y);
    const uint16_t h2 = to_bf16_bits(acc.z), h3 = to_bf16_bits(acc.w);
    uint2 hv, lv;
    hv.x = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
    hv.y = static_cast<uint32_t>(h2) | (static_cast<uint32_t>(h3) << 16);
    lv.x = pack_bf16x2(acc.x - bf16_bits_to_float(h0), acc.y - bf16_bits_to_float(h1));
    lv.y = pack_bf16x2(acc.z - bf16_bits_to_float(h2), acc.w - bf16_bits_to_float(h3));
    const size_t o = static_cast<size_t>(m0 + row) * p.r_pad + j0 + 4 * c4;
    *reinterpret_cast<uint2*>(p.t_hi + o) = hv;
    *reinterpret_cast<uint2*>(p.t_lo + o) = lv;
  }
  cluster_sync();  // no CTA leaves while a peer still reads its partial
}

// =====================================================================
// Kernel 3: fused main GEMM
// =====================================================================
struct MainParams {
  CUtensorMap tm_x;    // bf16 [M, K]       box {64, 128}, 128B swizzle
  CUtensorMap tm_q;    // u8   [N, K]       box {64, 128},  64B swizzle
  CUtensorMap tm_a;    // bf16 [N, r_pad]   box {64, 128}, 128B swizzle
  CUtensorMap tm_thi;  // bf16 [M, r_pad]   box {64, 128}, 128B swizzle
  CUtensorMap tm_tlo;  // bf16 [M, r_pad]
  CUtensorMap tm_y;    // bf16 [M, N]       box {32, 32},  no swizzle
  const float* scale;  // [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  int M, N, K, r_pad;
  int n_ftiles, n_ttiles;
  int lr_from_primary;  // 1: t is produced by the preceding kernel (wait on it)
  int withhold;         // debug: the TMA producer issues nothing
  Watch watch;
};

constexpr int kMainThreads = 320;  // 0: TMA, 1: MMA, 2-5: converters, 6-9: epilogue
constexpr int kSX = 6;             // x / A / t slots, 16 KB each
constexpr int kSQ = 8;             // Q slots, 8 KB each
constexpr int kNA = 8;             // widened-Q stages in TMEM, 32 columns each
constexpr int kXSlot = 128 * kBK * 2;
constexpr int kQSlot = 128 * kBK;
constexpr int kEpiBytes = 4 * 2 * 32 * 32 * 2;
constexpr int kTmemCols = 512;
constexpr int kColAccQ = 0, kColAccLR = 128, kColA = 256;

__host__ __device__ constexpr int main_smem_bytes() {
  return kSX * kXSlot + kSQ * kQSlot + kEpiBytes + 1024 /*align*/ + 512 /*barriers*/;
}

template <int kAct>
__global__ void __launch_bounds__(kMainThreads, 1) ll_main_kernel(const __grid_constant__ MainParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sx = smem;
  uint8_t* sq = sx + kSX * kXSlot;
  uint8_t* se = sq + kSQ * kQSlot;
  uint64_t* x_full = reinterpret_cast<uint64_t*>(se + kEpiBytes);
  uint64_t* x_empty = x_full + kSX;
  uint64_t* q_full = x_empty + kSX;
  uint64_t* q_empty = q_full + kSQ;
  uint64_t* a_full = q_empty + kSQ;
  uint64_t* a_empty = a_full + kNA;
  uint64_t* acc_full = a_empty + kNA;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.n_ftiles * p.n_ttiles;
  const int nK = (p.K + kBK - 1) / kBK;
  const int nR = (p.r_pad + kBK - 1) / kBK;  // columns past r_pad load as zeros

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSX; ++s) { mbar_init(&x_full[s], 1); mbar_init(&x_empty[s], 1); }
    for (int s = 0; s < kSQ; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 4); }
    for (int s = 0; s < kNA; ++s) { mbar_init(&a_full[s], 4); mbar_init(&a_empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_y);
    if (nR > 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_thi);
      tma_prefetch_desc(&p.tm_tlo);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && !p.withhold) {
      int xi = 0, qi = 0;
      uint32_t xph = 0, qph = 0;
      long long nx = 0, nq = 0;  // loads issued per ring
      bool ok = true, waited_primary = false;
      for (int T = blockIdx.x; T < n_tiles && ok; T += gridDim.x) {
        const int f0 = (T / p.n_ttiles) * 128;
        const int t0 = (T % p.n_ttiles) * 128;
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(&x_full[xi], kXSlot);
          tma_load_2d(sx + xi * kXSlot, &p.tm_x, &x_full[xi], kb * kBK, t0);
          ++nx;
          if (++xi == kSX) { xi = 0; xph ^= 1; }
          if (!mbar_wait(&q_empty[qi], qph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[qi], kQSlot);
          tma_load_2d(sq + qi * kQSlot, &p.tm_q, &q_full[qi], kb * kBK, f0);
          ++nq;
          if (++qi == kSQ) { qi = 0; qph ^= 1; }
        }
        if (!ok || nR == 0) continue;
        if (!waited_primary && p.lr_from_primary) {
          pdl_wait_primary();
          waited_primary = true;
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          const CUtensorMap* maps[3] = {&p.tm_a, &p.tm_thi, &p.tm_tlo};
          const int rows[3] = {f0, t0, t0};
#pragma unroll
          for (int w = 0; w < 3; ++w) {
            if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            mbar_arrive_expect_tx(&x_full[xi], kXSlot);
            tma_load_2d(sx + xi * kXSlot, maps[w], &x_full[xi], jb * kBK, rows[w]);
            ++nx;
            if (++xi == kSX) { xi = 0; xph ^= 1; }
          }
        }
      }
      if (!ok) {
        for (long long i = (nx > kSX ? nx - kSX : 0); i < nx; ++i)
          mbar_wait_drain(&x_full[i % kSX], static_cast<uint32_t>((i / kSX) & 1), p.watch);
        for (long long i = (nq > kSQ ? nq - kSQ : 0); i < nq; ++i)
          mbar_wait_drain(&q_full[i % kSQ], static_cast<uint32_t>((i / kSQ) & 1), p.watch);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      int xi = 0, ai = 0;
      uint32_t xph = 0, aph = 0, accph = 0;
      bool ok = true;
      const uint32_t d_q = tbase + kColAccQ, d_lr = tbase + kColAccLR;
      for (int T = blockIdx.x; T < n_tiles && ok; T += gridDim.x) {
        const int t0 = (T % p.n_ttiles) * 128;
        const int valid = min(128, p.M - t0);
        const uint32_t idesc = idesc_bf16(128, (valid + 15) & ~15);
        if (!mbar_wait(acc_empty, accph ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&a_full[ai], aph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          if (!mbar_wait(&x_full[xi], xph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sx + xi * kXSlot));
          const uint32_t at = tbase + kColA + ai * 32;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ts(d_q, at + kk * 8, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&x_empty[xi]);
          tc_commit(&a_empty[ai]);
          if (++xi == kSX) { xi = 0; xph ^= 1; }
          if (++ai == kNA) { ai = 0; aph ^= 1; }
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          int slot[3];
#pragma unroll
          for (int w = 0; w < 3; ++w) {
            if (!mbar_wait(&x_full[xi], xph, p.watch, kErrTimeoutMma)) { ok = false; break; }
            slot[w] = xi;
            if (++xi == kSX) { xi = 0; xph ^= 1; }
          }
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sx + slot[0] * kXSlot));
          const uint64_t hd = sdesc_kmajor_sw128(smem_u32(sx + slot[1] * kXSlot));
          const uint64_t ld = sdesc_kmajor_sw128(smem_u32(sx + slot[2] * kXSlot));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(d_lr, ad + 2 * kk, hd + 2 * kk, idesc, (jb | kk) != 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) mma_ss(d_lr, ad + 2 * kk, ld + 2 * kk, idesc, 1u);
#pragma unroll
          for (int w = 0; w < 3; ++w) tc_commit(&x_empty[slot[w]]);
        }
        if (!ok) break;
        tc_commit(acc_full);
        accph ^= 1;
      }
      // No MMA may still run when TMEM is released below.
      tc_commit(drain);
      mbar_wait_drain(drain, 0, p.watch);
    }
  } else if (warp < 6) {
    // --------------------------------------------- e4m3 -> bf16 into TMEM
    const int q = warp & 3;
    const int row = 32 * q + lane;  // feature row within the tile = TMEM lane
    const uint32_t tl = tbase + ((32u * q) << 16);
    int qi = 0, ai = 0;
    uint32_t qph = 0, aph = 0;
    bool ok = true;
    for (int T = blockIdx.x; T < n_tiles && ok; T += gridDim.x) {
      for (int kb = 0; kb < nK; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qi], qph, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        // The Q slot holds 128 rows of 64 codes with the 64-byte swizzle:
        // 16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3).
        const uint8_t* rb = sq + qi * kQSlot + row * 64;
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(rb + 16 * (j ^ ((row >> 1) & 3)));
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[qi]);
        if (++qi == kSQ) { qi = 0; qph ^= 1; }
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e4m3x4_to_bf16x4(v[j].x, w[8 * j + 0], w[8 * j + 1]);
          e4m3x4_to_bf16x4(v[j].y, w[8 * j + 2], w[8 * j + 3]);
          e4m3x4_to_bf16x4(v[j].z, w[8 * j + 4], w[8 * j + 5]);
          e4m3x4_to_bf16x4(v[j].w, w[8 * j + 6], w[8 * j + 7]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[ai], aph ^ 1, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        tc_fence_after();
        tmem_st32_wait(tl + kColA + ai * 32, w);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[ai]);
        if (++ai == kNA) { ai = 0; aph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int frow = 32 * q + lane;
    const uint32_t tl = tbase + ((32u * q) << 16);
    uint16_t* stage = reinterpret_cast<uint16_t*>(se + (warp - 6) * (2 * 32 * 32 * 2));
    int eb = 0;
    uint32_t accph = 0;
    const bool has_lr = nR > 0;
    for (int T = blockIdx.x; T < n_tiles; T += gridDim.x) {
      const int f0 = (T / p.n_ttiles) * 128;
      const int t0 = (T % p.n_ttiles) * 128;
      const int valid = min(128, p.M - t0);
      const int f = f0 + frow;
      const float s = f < p.N ? p.scale[f] : 0.f;
      const float b = (p.bias != nullptr && f < p.N) ? bf16_bits_to_float(p.bias[f]) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, accph, p.watch, kErrTimeoutEpilogue))) break;
      tc_fence_after();
      const bool store_rows = f0 + 32 * q < p.N;
      for (int c = 0; c < valid; c += 32) {
        uint32_t aq[32], al[32];
        if (has_lr) {
          tmem_ld32x2_wait(tl + kColAccQ + c, aq, tl + kColAccLR + c, al);
        } else {
          tmem_ld32_wait(tl + kColAccQ + c, aq);
#pragma unroll
          for (int i = 0; i < 32; ++i) al[i] = 0u;
        }
        if (lane == 0) tma_store_wait_read<1>();
        __syncwarp();
        uint16_t* st = stage + eb * (32 * 32);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float v = fmaf(s, __uint_as_float(aq[i]), __uint_as_float(al[i]) + b);
          st[i * 32 + lane] = to_bf16_bits(epi_act<kAct>(v));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && store_rows) {
          tma_store_2d(&p.tm_y, st, f0 + 32 * q, t0 + c);
        }
        if (lane == 0) tma_store_commit();
        eb ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      accph ^= 1;
    }
    if (lane == 0) tma_store_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Flags any NaN code (0x7F or 0xFF) of an e4m3fn array.
__global__ void ll_nan_scan_kernel(const uint8_t* __restrict__ q, size_t n, int* __restrict__ flag) {
  const size_t n16 = n / 16;
  int found = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(q)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t m = w[j] & 0x7F7F7F7Fu;
      // a byte equals 0x7F after masking the sign iff it is a NaN code
      const uint32_t x = m ^ 0x7F7F7F7Fu;
      found |= ((x - 0x01010101u) & ~x & 0x80808080u) != 0;
    }
  }
  for (size_t i = n16 * 16 + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    found |= (q[i] & 0x7F) == 0x7F;
  if (found) atomicOr(flag, 1);
}

}  // namespace llk
