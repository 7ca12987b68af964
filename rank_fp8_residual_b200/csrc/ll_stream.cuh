// Small-M streaming kernel (sm_100a) of the LiteLinear forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// for M <= 64 tokens.  At these sizes the forward is bound by reading Q
// (N*K bytes) and A (2*N*r bytes) from HBM once, so the kernel is shaped to
// stream them: every CTA owns 128 output features (one tile; persistent
// CTAs stride over tiles when there are more tiles than SMs) and pulls its
// Q rows in 32 KB groups (4 K chunks of 64 codes) through a four-slot
// ring.  The tokens (padded to Mt = 16, 32, 48 or 64) are the MMA N side,
// so one MMA covers all of them:
//
//   acc_Q  [128 features x Mt tokens] += Qdec[128 x 16] * x[Mt x 16]^T
//                                        (tcgen05 TS form: Qdec in TMEM)
//   acc_LR [128 x Mt]                 += A[128 x 16] * (t_hi + t_lo)[Mt x 16]^T
//                                        (SS form, exact A)
//   y[m, n] = bf16( scale[n] * acc_Q + acc_LR + bias[n] )
//
// t = x B^T comes from ll_lrdown_kernel, which runs beside this kernel on
// the SMs this grid leaves free (programmatic dependent launch); the x
// producer waits for it only after the tile's last x load, so the residual
// stream never waits for t.
//
// The widened residual goes through TMEM in stages of two K chunks (64
// columns), four stages deep.  Each converter warp widens one full chunk
// row (64 codes) per stage, and two teams of eight converter warps take
// alternate stages, so four converter warps share each SM sub-partition
// and hide one another's shared-memory, barrier and TMEM-store latency.
//
// Warp roles (19 warps): 0 TMA producer of Q, 1 MMA issuer (also
// allocates TMEM), 2-17 converters that, after the tile's last MMA, also
// run the epilogue straight from TMEM to global memory (each warp stores
// 32 consecutive features per token: 64-byte segments), 18 TMA producer of
// x and of the low-rank A / t chunks.  The two producers are separate so
// that the Q stream from HBM runs ahead of the x ring, which only frees up
// as fast as the MMAs consume it.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

struct StreamParams {
  CUtensorMap tm_x;    // bf16 x: 3-D {64, M, K/64} box {64, Mt, 4}, or 2-D [M, K] box {64, Mt}; 128B swizzle
  CUtensorMap tm_q;    // u8 Q:   3-D {64, N, K/64} box {64, 128, 4}, or 2-D [N, K] box {64, 128}; 64B swizzle
  CUtensorMap tm_a;    // bf16 A [N, r_pad] box {64, 128}, 128B swizzle
  CUtensorMap tm_thi;  // bf16 t_hi [M, r_pad] box {64, Mt}, 128B swizzle
  CUtensorMap tm_tlo;  // bf16 t_lo [M, r_pad]
  const float* scale;    // [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  uint16_t* y;           // [M, N] bf16 bits
  int M, N, K, r_pad;
  int Mt;                // MMA N: tokens padded to a multiple of 16, 16..64
  int n_ftiles;
  int dims3;             // 1: one 3-D load per group of 4 chunks; 0: four 2-D loads
  int lr_from_primary;   // 1: t is produced by the preceding kernel
  int withhold;          // debug: the TMA producers issue nothing
  Watch watch;
};

constexpr int kStConvWarps = 16;  // two teams of 8; team t widens the stages of parity t
constexpr int kStXWarp = 2 + kStConvWarps;           // warp of the x / low-rank producer
constexpr int kStThreads = 32 * (3 + kStConvWarps);  // Q producer, MMA, converters, x producer
constexpr int kStGroup = 4;               // K chunks per Q / x slot
constexpr int kStSQ = 4;                  // Q slots (32 KB each)
constexpr int kStSX = 3;                  // x slots (also A / t chunks of the low-rank phase)
constexpr int kStNA = 4;                  // widened-Q stages in TMEM, 2 chunks = 64 columns each
constexpr int kStQChunk = 128 * kBK;      // 8 KB: 128 rows x 64 codes
constexpr int kStQSlot = kStGroup * kStQChunk;
constexpr int kStMaxMt = 64;
constexpr int kStColLR = 64;              // TMEM column of acc_LR
constexpr int kStColA = 128;              // TMEM column of the first widened-Q stage

__host__ __device__ constexpr int st_round1k(int v) { return (v + 1023) / 1024 * 1024; }
// x slot: one group of x (Mt x 256 bf16), or one low-rank chunk (A 128 x 64,
// t_hi and t_lo Mt x 64).
__host__ __device__ constexpr int st_xslot_bytes(int Mt) {
  return st_round1k(Mt * 128 * kStGroup > 16384 + 2 * Mt * 128 ? Mt * 128 * kStGroup : 16384 + 2 * Mt * 128);
}
__host__ __device__ constexpr int st_smem_bytes(int Mt) {
  return kStSQ * kStQSlot + kStSX * st_xslot_bytes(Mt) + 1024 /*align*/ + 512 /*barriers*/;
}
__host__ __device__ constexpr int st_smem_max() { return st_smem_bytes(kStMaxMt); }

template <int kAct>
__global__ void __launch_bounds__(kStThreads, 1) ll_stream_kernel(const __grid_constant__ StreamParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int xslot = st_xslot_bytes(p.Mt);
  uint8_t* sq = smem;
  uint8_t* sx = sq + kStSQ * kStQSlot;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sx + kStSX * xslot);
  uint64_t* q_empty = q_full + kStSQ;
  uint64_t* x_full = q_empty + kStSQ;
  uint64_t* x_empty = x_full + kStSX;
  uint64_t* a_full = x_empty + kStSX;
  uint64_t* a_empty = a_full + kStNA;
  uint64_t* acc_full = a_empty + kStNA;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nKc = (p.K + kBK - 1) / kBK;         // 64-wide K chunks
  const int nG = (nKc + kStGroup - 1) / kStGroup;  // groups; chunks past K load as zeros
  const int nR = (p.r_pad + kBK - 1) / kBK;       // 64-wide rank chunks (past r_pad: zeros)
  const int tbytes = p.Mt * 128;                 // one Mt x 64 bf16 tile
  const int xbytes = tbytes * kStGroup;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStSQ; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], kStConvWarps); }
    for (int s = 0; s < kStSX; ++s) { mbar_init(&x_full[s], 1); mbar_init(&x_empty[s], 1); }
    for (int s = 0; s < kStNA; ++s) { mbar_init(&a_full[s], kStConvWarps / 2); mbar_init(&a_empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kStConvWarps);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_q);
    if (nR > 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_thi);
      tma_prefetch_desc(&p.tm_tlo);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA: Q (HBM)
    // Runs ahead of everything else by up to kStSQ groups.
    if (lane == 0 && !p.withhold) {
      int qi = 0;
      uint32_t qph = 0;
      long long nq = 0;
      bool ok = true;
      for (int T = blockIdx.x; T < p.n_ftiles && ok; T += gridDim.x) {
        const int f0 = T * 128;
        for (int g = 0; g < nG; ++g) {
          if (!mbar_wait(&q_empty[qi], qph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          uint8_t* dst = sq + qi * kStQSlot;
          mbar_arrive_expect_tx(&q_full[qi], kStQSlot);
          if (p.dims3) {
            tma_load_3d(dst, &p.tm_q, &q_full[qi], 0, f0, g * kStGroup);
          } else {
#pragma unroll
            for (int i = 0; i < kStGroup; ++i)
              tma_load_2d(dst + i * kStQChunk, &p.tm_q, &q_full[qi], (g * kStGroup + i) * kBK, f0);
          }
          ++nq;
          if (++qi == kStSQ) { qi = 0; qph ^= 1; }
        }
      }
      if (!ok) {
        // Let every load already issued land before the CTA can exit.
        for (long long i = (nq > kStSQ ? nq - kStSQ : 0); i < nq; ++i)
          mbar_wait_drain(&q_full[i % kStSQ], static_cast<uint32_t>((i / kStSQ) & 1), p.watch);
      }
    }
  } else if (warp == kStXWarp) {
    // ----------------------------------- TMA: x, then A and t chunks (L2)
    if (lane == 0 && !p.withhold) {
      int xi = 0;
      uint32_t xph = 0;
      long long nx = 0;
      bool ok = true, waited_primary = false;
      for (int T = blockIdx.x; T < p.n_ftiles && ok; T += gridDim.x) {
        const int f0 = T * 128;
        for (int g = 0; g < nG; ++g) {
          if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          uint8_t* dst = sx + xi * xslot;
          mbar_arrive_expect_tx(&x_full[xi], xbytes);
          if (p.dims3) {
            tma_load_3d(dst, &p.tm_x, &x_full[xi], 0, 0, g * kStGroup);
          } else {
#pragma unroll
            for (int i = 0; i < kStGroup; ++i)
              tma_load_2d(dst + i * tbytes, &p.tm_x, &x_full[xi], (g * kStGroup + i) * kBK, 0);
          }
          ++nx;
          if (++xi == kStSX) { xi = 0; xph ^= 1; }
        }
        if (!ok || nR == 0) continue;
        if (!waited_primary && p.lr_from_primary) {
          pdl_wait_primary();
          waited_primary = true;
        }
        for (int jb = 0; jb < nR; ++jb) {
          if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          uint8_t* st = sx + xi * xslot;
          mbar_arrive_expect_tx(&x_full[xi], 16384 + 2 * tbytes);
          tma_load_2d(st, &p.tm_a, &x_full[xi], jb * kBK, f0);
          tma_load_2d(st + 16384, &p.tm_thi, &x_full[xi], jb * kBK, 0);
          tma_load_2d(st + 16384 + tbytes, &p.tm_tlo, &x_full[xi], jb * kBK, 0);
          ++nx;
          if (++xi == kStSX) { xi = 0; xph ^= 1; }
        }
      }
      if (!ok) {
        for (long long i = (nx > kStSX ? nx - kStSX : 0); i < nx; ++i)
          mbar_wait_drain(&x_full[i % kStSX], static_cast<uint32_t>((i / kStSX) & 1), p.watch);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      int xi = 0, ai = 0;
      uint32_t xph = 0, aph = 0, accph = 0;
      bool ok = true;
      const uint32_t d_q = tbase, d_lr = tbase + kStColLR;
      const uint32_t idesc = idesc_bf16(128, p.Mt);
      for (int T = blockIdx.x; T < p.n_ftiles && ok; T += gridDim.x) {
        if (!mbar_wait(acc_empty, accph ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        for (int g = 0; g < nG && ok; ++g) {
          if (!mbar_wait(&x_full[xi], xph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          const uint32_t xs = smem_u32(sx + xi * xslot);
          for (int h2 = 0; h2 < kStGroup / 2; ++h2) {
            if (!mbar_wait(&a_full[ai], aph, p.watch, kErrTimeoutMma)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              const int ch = 2 * h2 + sub;  // chunk within the group
              const uint64_t bd = sdesc_kmajor_sw128(xs + ch * tbytes);
              const uint32_t at = tbase + kStColA + ai * 64 + sub * 32;
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                mma_ts(d_q, at + kk * 8, bd + 2 * kk, idesc, (g | ch | kk) != 0 ? 1u : 0u);
            }
            tc_commit(&a_empty[ai]);
            if (++ai == kStNA) { ai = 0; aph ^= 1; }
          }
          if (!ok) break;
          tc_commit(&x_empty[xi]);
          if (++xi == kStSX) { xi = 0; xph ^= 1; }
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          if (!mbar_wait(&x_full[xi], xph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(sx + xi * xslot);
          const uint64_t ad = sdesc_kmajor_sw128(st);
          const uint64_t hd = sdesc_kmajor_sw128(st + 16384);
          const uint64_t ld = sdesc_kmajor_sw128(st + 16384 + tbytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(d_lr, ad + 2 * kk, hd + 2 * kk, idesc, (jb | kk) != 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) mma_ss(d_lr, ad + 2 * kk, ld + 2 * kk, idesc, 1u);
          tc_commit(&x_empty[xi]);
          if (++xi == kStSX) { xi = 0; xph ^= 1; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        accph ^= 1;
      }
      // No MMA may still run when TMEM is released below.
      tc_commit(drain);
      mbar_wait_drain(drain, 0, p.watch);
    }
  } else if (warp < 2 + kStConvWarps) {
    // ------------------------- e4m3 -> bf16 into TMEM stages, then epilogue
    // Team t (warps 2+8t .. 9+8t) widens the stage of parity t of every
    // group (chunks 2t and 2t+1); within a team, warp (q, par) takes lane
    // quadrant q and chunk 2t+par, one full 64-code row per lane.
    const int cw = warp - 2;
    const int team = cw >> 3;
    const int q = warp & 3;
    const int par = (cw >> 2) & 1;
    const int row = 32 * q + lane;     // feature row within the tile = TMEM lane
    const int sw = (row >> 1) & 3;     // 64-byte swizzle phase of the row
    const uint32_t tl = tbase + ((32u * q) << 16);
    const bool has_lr = nR > 0;
    const int chunk = 2 * team + par;  // chunk of each group this warp widens
    int qi = 0, ai = team;             // stage index: 2g + team (mod kStNA)
    uint32_t qph = 0, aph = 0, accph = 0;
    bool ok = true;
    for (int T = blockIdx.x; T < p.n_ftiles && ok; T += gridDim.x) {
      for (int g = 0; g < nG; ++g) {
        if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qi], qph, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        uint4 v[4];
        const uint8_t* rb = sq + qi * kStQSlot + chunk * kStQChunk + row * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(rb + 16 * (j ^ sw));
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[qi]);
        if (++qi == kStSQ) { qi = 0; qph ^= 1; }
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e4m3x4_to_bf16x4(v[j].x, w[8 * j + 0], w[8 * j + 1]);
          e4m3x4_to_bf16x4(v[j].y, w[8 * j + 2], w[8 * j + 3]);
          e4m3x4_to_bf16x4(v[j].z, w[8 * j + 4], w[8 * j + 5]);
          e4m3x4_to_bf16x4(v[j].w, w[8 * j + 6], w[8 * j + 7]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[ai], aph ^ 1, p.watch, kErrTimeoutConvert))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32_wait(tl + kStColA + ai * 64 + 32 * par, w);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[ai]);
        ai += 2;
        if (ai >= kStNA) { ai -= kStNA; aph ^= 1; }
      }
      if (!ok) break;

      // Epilogue: TMEM lane = feature, column = token.  The four warps of
      // a lane quadrant take the 16-token column blocks 2*team+par mod 4.
      const int f = T * 128 + row;
      const float sc = f < p.N ? p.scale[f] : 0.f;
      const float b = (p.bias != nullptr && f < p.N) ? bf16_bits_to_float(p.bias[f]) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, accph, p.watch, kErrTimeoutEpilogue))) break;
      accph ^= 1;
      tc_fence_after();
      for (int cb = 16 * chunk; cb < p.Mt; cb += 64) {
        uint32_t aq[16], al[16];
        tmem_ld16x2_wait(tl + cb, aq, tl + kStColLR + cb, al);
        if (f < p.N) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int m = cb + i;
            const float lr = has_lr ? __uint_as_float(al[i]) : 0.f;
            if (m < p.M) p.y[static_cast<size_t>(m) * p.N + f] = to_bf16_bits(epi_act<kAct>(fmaf(sc, __uint_as_float(aq[i]), lr + b)));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace llk
