// Large-M fused kernel (sm_100a) of the LiteLinear forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// evaluated per output row n as
//
//     y[m, n] = s[n] * ( sum_k Q[n,k] x[m,k] + sum_j A'[n,j] t[m,j] ) + bias[n]
//
// with t = x B^T (from ll_lrdown_kernel, carried as bf16 t_hi + t_lo) and
// A' = A / s[n] carried as bf16 A'_hi + A'_lo (prepared once when the
// weights are set).  Multiplying out, s*A'*t = A*t, so the single fp32
// accumulator holds both terms and the epilogue applies s[n] and the bias
// once.  The low-rank product uses three bf16 MMAs per K step
// (A'_hi t_hi + A'_hi t_lo + A'_lo t_hi); the dropped A'_lo t_lo term and
// the two pair splittings leave a relative error of order 2^-16 on the
// low-rank term.  Rows with s[n] == 0 use s = 1 and an all-zero residual row
// (exact, since 0 * (x Q^T) = 0).
//
// Tile: 128 output features (MMA M, TMEM lanes) x bt tokens (MMA N, TMEM
// columns; bt <= 256, a multiple of 16 chosen per call so that the tiles
// fill the SMs in as few equal waves as possible).  Q is the MMA A operand:
// eight converter warps widen the e4m3fn codes exactly to bf16 and store
// them into TMEM stages of two K steps (64 columns); x is the B operand,
// staged by TMA, whose two chunks of a stage complete on that stage's TMEM
// barrier, so the MMA issuer waits once per eight MMAs.  Persistent CTAs take tiles from a device-wide counter in a
// grouped raster order (8 token tiles per group) so that the tiles in flight
// share their x and Q slabs in L2.  Every tile, the first included, comes
// from that counter.
//
// Warp roles (27 warps): 0 TMA producer of Q + tile scheduler, 1 MMA issuer
// (also allocates TMEM), 2-17 converters in two teams of eight that take
// alternate stages (lane quadrant w%4, K step parity within a stage), so
// four converter warps share each SM sub-partition and hide one another's
// shared-memory, barrier and TMEM-store latency, 18-25 epilogue (lane
// quadrant w%4, two warps per quadrant on alternate 32-token blocks, so the
// accumulator is free for the next tile sooner), 26 TMA producer of x and
// of the low-rank A' / t chunks.  The two producers are
// separate so that each ring runs ahead on its own.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

struct TcParams {
  CUtensorMap tm_x;    // bf16 [M, K]       box {64, bt},   128B swizzle
  CUtensorMap tm_q;    // u8   [N, K]       3-D {64, N, K/64} box {64, 128, 2}, or 2-D box {64, 128}; 64B swizzle
  CUtensorMap tm_ahi;  // bf16 [N, r_pad]   box {klr, 128}, 128B (klr 64) / 64B (klr 32) swizzle
  CUtensorMap tm_alo;  // bf16 [N, r_pad]
  CUtensorMap tm_thi;  // bf16 [M, r_pad]   box {klr, bt}
  CUtensorMap tm_tlo;  // bf16 [M, r_pad]
  CUtensorMap tm_y;    // bf16 [M, N]       box {32, 32},    no swizzle
  const float* scale;    // effective per-row scale [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  int* sched;            // [2]: tile counter, finished-CTA counter (0 between launches)
  int M, N, K, r_pad, klr;
  int bt;                // tokens per tile (multiple of 16, <= 256)
  int n_ftiles, n_ttiles;
  int q3;                // 1: one 3-D Q load per stage; 0: two 2-D loads
  int lr_from_primary;
  int withhold;
  Watch watch;
};

constexpr int kTcConvWarps = 16;  // two teams of 8; team t widens the stages of parity t
constexpr int kTcEpiWarps = 8;   // two per lane quadrant, alternate 32-token blocks
constexpr int kTcXWarp = 2 + kTcConvWarps + kTcEpiWarps;  // x / low-rank producer
constexpr int kTcThreads = 32 * (kTcXWarp + 1);
constexpr int kTcMaxBT = 256;               // tokens per tile, at most
constexpr int kTcSX = 5;                    // 32 KB slots: x chunks, A'/t chunks
constexpr int kTcSQ = 2;                    // 16 KB slots: Q, two K steps each
constexpr int kTcNA = 4;                    // widened-Q stages in TMEM (two K steps, 64 columns each)
constexpr int kTcXSlot = kTcMaxBT * kBK * 2;  // 32768
constexpr int kTcQChunk = 128 * kBK;        // 8192: 128 rows x 64 codes
constexpr int kTcQSlot = 2 * kTcQChunk;
constexpr int kTcEpi = kTcEpiWarps * 2 * 32 * 32 * 2;
constexpr int kTcGroup = 8;                 // token tiles per raster group
constexpr int kTcTileRing = 2;
constexpr int kTcColA = 256;                // TMEM column of the first widened-Q stage
// Consumers of a scheduled tile: MMA, converters, epilogue, x producer.
constexpr int kTcTileUsers = 1 + kTcConvWarps + kTcEpiWarps + 1;

__host__ __device__ constexpr int tc_smem_bytes() {
  return kTcSX * kTcXSlot + kTcSQ * kTcQSlot + kTcEpi + 1024 + 512;
}

__device__ __forceinline__ void tc_tile_coords(int T, int n_ftiles, int n_ttiles, int bt, int& f0, int& t0) {
  const int per_group = kTcGroup * n_ftiles;
  const int g = T / per_group;
  const int first_tt = g * kTcGroup;
  const int gsize = min(kTcGroup, n_ttiles - first_tt);
  const int idx = T - g * per_group;
  f0 = (idx / gsize) * 128;
  t0 = (first_tt + idx % gsize) * bt;
}

template <int kAct>
__global__ void __launch_bounds__(kTcThreads, 1) ll_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sx = smem;
  uint8_t* sq = sx + kTcSX * kTcXSlot;
  uint8_t* se = sq + kTcSQ * kTcQSlot;
  uint64_t* x_full = reinterpret_cast<uint64_t*>(se + kTcEpi);
  uint64_t* x_empty = x_full + kTcSX;
  uint64_t* q_full = x_empty + kTcSX;
  uint64_t* q_empty = q_full + kTcSQ;
  uint64_t* a_full = q_empty + kTcSQ;
  uint64_t* a_empty = a_full + kTcNA;
  uint64_t* acc_full = a_empty + kTcNA;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* tile_full = acc_empty + 1;
  uint64_t* tile_empty = tile_full + kTcTileRing;
  uint64_t* drain = tile_empty + kTcTileRing;
  int* tile_slot = reinterpret_cast<int*>(drain + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_slot + kTcTileRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.n_ftiles * p.n_ttiles;
  const int nK = (p.K + kBK - 1) / kBK;
  const int nS = (nK + 1) / 2;  // stages of two K steps (a step past K loads as zeros)
  const int nR = p.r_pad / p.klr;
  const int klr = p.klr;
  const int bt = p.bt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcSX; ++s) { mbar_init(&x_full[s], 1); mbar_init(&x_empty[s], 1); }
    // A Q slot and a TMEM stage each hold one stage, which one team reads / writes.
    for (int s = 0; s < kTcSQ; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], kTcConvWarps / 2); }
    // a_full[stage]: the converter team's eight arrivals plus the x
    // producer's (with the transaction bytes of the stage's two x chunks),
    // so one wait tells the MMA issuer that both operands are in place.
    for (int s = 0; s < kTcNA; ++s) { mbar_init(&a_full[s], kTcConvWarps / 2 + 1); mbar_init(&a_empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kTcEpiWarps);
    for (int s = 0; s < kTcTileRing; ++s) {
      mbar_init(&tile_full[s], 1);
      mbar_init(&tile_empty[s], kTcTileUsers);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_y);
    if (nR > 0) {
      tma_prefetch_desc(&p.tm_ahi);
      tma_prefetch_desc(&p.tm_alo);
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
    // --------------------------------------------- TMA: Q + tile scheduler
    if (lane == 0) {
      int qi = 0, ti = 0;
      uint32_t qph = 0, tph = 0;
      long long nq = 0;
      bool ok = true;
      for (;;) {
        if (!mbar_wait(&tile_empty[ti], tph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
        // Every tile, the first included, comes from the shared counter, so
        // a CTA that starts late (its SM still busy with the kernel before)
        // simply takes fewer tiles.
        const int T = atomicAdd(&p.sched[0], 1);
        const bool live = T < n_tiles;
        *reinterpret_cast<volatile int*>(&tile_slot[ti]) = live ? T : -1;
        mbar_arrive(&tile_full[ti]);
        if (++ti == kTcTileRing) { ti = 0; tph ^= 1; }
        if (!live) break;
        if (p.withhold) { ok = false; break; }  // debug: no loads, the consumers time out
        int f0, t0;
        tc_tile_coords(T, p.n_ftiles, p.n_ttiles, bt, f0, t0);
        for (int s = 0; s < nS; ++s) {
          if (!mbar_wait(&q_empty[qi], qph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          uint8_t* dst = sq + qi * kTcQSlot;
          mbar_arrive_expect_tx(&q_full[qi], kTcQSlot);
          if (p.q3) {
            tma_load_3d(dst, &p.tm_q, &q_full[qi], 0, f0, 2 * s);
          } else {
            tma_load_2d(dst, &p.tm_q, &q_full[qi], 2 * s * kBK, f0);
            tma_load_2d(dst + kTcQChunk, &p.tm_q, &q_full[qi], (2 * s + 1) * kBK, f0);
          }
          ++nq;
          if (++qi == kTcSQ) { qi = 0; qph ^= 1; }
        }
        if (!ok) break;
      }
      if (!ok) {
        for (long long i = (nq > kTcSQ ? nq - kTcSQ : 0); i < nq; ++i)
          mbar_wait_drain(&q_full[i % kTcSQ], static_cast<uint32_t>((i / kTcSQ) & 1), p.watch);
      }
      // The last CTA to finish resets the scheduler for the next launch.
      __threadfence();
      if (atomicAdd(&p.sched[1], 1) == static_cast<int>(gridDim.x) - 1) {
        atomicExch(&p.sched[0], 0);
        atomicExch(&p.sched[1], 0);
      }
    }
  } else if (warp == kTcXWarp) {
    // --------------------------------- TMA: x, then A' and t chunks (L2)
    if (lane == 0) {
      int xi = 0, ti = 0;
      uint32_t xph = 0, tph = 0;
      uint32_t lr_ph = 0;  // per-slot phase bits of x_full (used by the low-rank chunks only)
      long long nx = 0;    // low-rank loads issued (on x_full)
      long long gsx = 0;   // residual stages issued (on a_full)
      long long pend_s = 0;  // residual stages whose loads were issued
      bool ok = true, waited_primary = false;
      const uint32_t x_bytes = static_cast<uint32_t>(bt) * kBK * 2u;
      const uint32_t a_bytes = 128u * klr * 2u;
      const uint32_t t_bytes = static_cast<uint32_t>(bt) * klr * 2u;
      for (;;) {
        if (!mbar_wait(&tile_full[ti], tph, p.watch, kErrTimeoutProducer)) { ok = false; break; }
        const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
        mbar_arrive(&tile_empty[ti]);
        if (++ti == kTcTileRing) { ti = 0; tph ^= 1; }
        if (T < 0) break;
        if (p.withhold) { ok = false; break; }
        int f0, t0;
        tc_tile_coords(T, p.n_ftiles, p.n_ttiles, bt, f0, t0);
        // Residual stages: the two x chunks of stage s go into the next two
        // slots and complete on the stage's a_full barrier.
        for (int s = 0; s < nS && ok; ++s) {
          int slot[2];
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            slot[h] = xi;
            if (++xi == kTcSX) { xi = 0; xph ^= 1; }
          }
          if (!ok) break;
          uint64_t* bar = &a_full[gsx % kTcNA];
          mbar_arrive_expect_tx(bar, 2 * x_bytes);
          tma_load_2d(sx + slot[0] * kTcXSlot, &p.tm_x, bar, 2 * s * kBK, t0);
          tma_load_2d(sx + slot[1] * kTcXSlot, &p.tm_x, bar, (2 * s + 1) * kBK, t0);
          ++gsx;
          pend_s = gsx;
        }
        if (ok && nR > 0 && !waited_primary && p.lr_from_primary) {
          pdl_wait_primary();
          waited_primary = true;
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          // slot 1: A'_hi | A'_lo chunk; slot 2: t_hi chunk; slot 3: t_lo chunk
          const CUtensorMap* maps[3] = {&p.tm_ahi, &p.tm_thi, &p.tm_tlo};
          for (int w = 0; w < 3; ++w) {
            if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            uint64_t* bar = &x_full[xi];
            if (w == 0) {
              mbar_arrive_expect_tx(bar, 2 * a_bytes);
              tma_load_2d(sx + xi * kTcXSlot, &p.tm_ahi, bar, jb * klr, f0);
              tma_load_2d(sx + xi * kTcXSlot + a_bytes, &p.tm_alo, bar, jb * klr, f0);
            } else {
              mbar_arrive_expect_tx(bar, t_bytes);
              tma_load_2d(sx + xi * kTcXSlot, maps[w], bar, jb * klr, t0);
            }
            ++nx;
            lr_ph ^= 1u << xi;
            if (++xi == kTcSX) { xi = 0; xph ^= 1; }
          }
        }
        if (!ok) break;
      }
      if (!ok && (pend_s > 0 || nx > 0)) {
        // Loads already issued must land before the CTA exits.  Residual
        // chunks complete on a_full, which also counts the converters (who
        // may have left), so instead of waiting on it wait a bounded settle
        // time, far above any load latency.
        const uint64_t c0 = clock_cycles();
        while (clock_cycles() - c0 < 400000ull) {  // >= 200 us at any clock up to 2 GHz
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      int xi = 0, ai = 0, ti = 0;
      uint32_t xph = 0, aph = 0, accph = 0, tph = 0;
      uint32_t lr_ph = 0;  // per-slot phase bits of x_full (low-rank chunks only)
      bool ok = true;
      const uint32_t a_bytes = 128u * klr * 2u;
      for (;;) {
        if (!mbar_wait(&tile_full[ti], tph, p.watch, kErrTimeoutMma)) break;
        const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
        mbar_arrive(&tile_empty[ti]);
        if (++ti == kTcTileRing) { ti = 0; tph ^= 1; }
        if (T < 0) break;
        int f0, t0;
        tc_tile_coords(T, p.n_ftiles, p.n_ttiles, bt, f0, t0);
        const int valid = min(bt, p.M - t0);
        const uint32_t idesc = idesc_bf16(128, (valid + 15) & ~15);
        if (!mbar_wait(acc_empty, accph ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        for (int s = 0; s < nS && ok; ++s) {
          // One wait per stage: converted Q (team) and both x chunks (TMA).
          if (!mbar_wait(&a_full[ai], aph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sx + xi * kTcXSlot));
            const uint32_t at = tbase + kTcColA + ai * 64 + sub * 32;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_ts(tbase, at + kk * 8, bd + 2 * kk, idesc, (s | sub | kk) != 0 ? 1u : 0u);
            tc_commit(&x_empty[xi]);
            if (++xi == kTcSX) { xi = 0; xph ^= 1; }
          }
          tc_commit(&a_empty[ai]);
          if (++ai == kTcNA) { ai = 0; aph ^= 1; }
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          int slot[3];
          for (int w = 0; w < 3; ++w) {
            if (!mbar_wait(&x_full[xi], (lr_ph >> xi) & 1u, p.watch, kErrTimeoutMma)) { ok = false; break; }
            lr_ph ^= 1u << xi;
            slot[w] = xi;
            if (++xi == kTcSX) { xi = 0; xph ^= 1; }
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(sx + slot[0] * kTcXSlot);
          const uint32_t sh = smem_u32(sx + slot[1] * kTcXSlot);
          const uint32_t sl = smem_u32(sx + slot[2] * kTcXSlot);
          uint64_t ah, al, th, tl;
          if (klr == 64) {
            ah = sdesc_kmajor_sw128(sa); al = sdesc_kmajor_sw128(sa + a_bytes);
            th = sdesc_kmajor_sw128(sh); tl = sdesc_kmajor_sw128(sl);
          } else {
            ah = sdesc_kmajor_sw64(sa); al = sdesc_kmajor_sw64(sa + a_bytes);
            th = sdesc_kmajor_sw64(sh); tl = sdesc_kmajor_sw64(sl);
          }
          for (int kk = 0; kk < klr / 16; ++kk) {
            mma_ss(tbase, ah + 2 * kk, th + 2 * kk, idesc, 1u);
            mma_ss(tbase, ah + 2 * kk, tl + 2 * kk, idesc, 1u);
            mma_ss(tbase, al + 2 * kk, th + 2 * kk, idesc, 1u);
          }
          for (int w = 0; w < 3; ++w) tc_commit(&x_empty[slot[w]]);
        }
        if (!ok) break;
        tc_commit(acc_full);
        accph ^= 1;
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0, p.watch);
    }
  } else if (warp < 2 + kTcConvWarps) {
    // ----------------------------------------- e4m3 -> bf16 into TMEM stages
    // Stages are numbered across this CTA's tiles (g); team t takes the
    // stages g = t (mod 2).  Within a team, warp (q, par) widens K step
    // 2s + par of the stage for the rows of lane quadrant q: one full
    // 64-code row chunk per lane.  Stage g uses Q slot g mod kTcSQ and
    // TMEM stage g mod kTcNA, each in the phase of its own lap.
    const int cw = warp - 2;
    const int team = cw >> 3;
    const int q = warp & 3;
    const int par = (cw >> 2) & 1;
    const int row = 32 * q + lane;              // feature row within the tile
    const int sw = (row >> 1) & 3;              // 64-byte swizzle phase of the row
    const uint32_t tl = tbase + ((32u * q) << 16) + kTcColA + 32 * par;
    int ti = 0;
    uint32_t tph = 0;
    long long gs = 0;  // stages of this CTA before the current tile
    bool ok = true;
    for (;;) {
      if (!__all_sync(0xffffffffu, mbar_wait(&tile_full[ti], tph, p.watch, kErrTimeoutConvert))) break;
      const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&tile_empty[ti]);
      if (++ti == kTcTileRing) { ti = 0; tph ^= 1; }
      if (T < 0) break;
      for (long long g = gs + ((team - gs) & 1); g < gs + nS; g += 2) {
        const int qslot = static_cast<int>(g % kTcSQ);
        const uint32_t qph = static_cast<uint32_t>((g / kTcSQ) & 1);
        const int slot = static_cast<int>(g % kTcNA);  // TMEM stage
        const uint32_t ph = static_cast<uint32_t>((g / kTcNA) & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qslot], qph, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        uint4 v[4];
        const uint8_t* rb = sq + qslot * kTcQSlot + par * kTcQChunk + row * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(rb + 16 * (j ^ sw));
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[qslot]);
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e4m3x4_to_bf16x4(v[j].x, w[8 * j + 0], w[8 * j + 1]);
          e4m3x4_to_bf16x4(v[j].y, w[8 * j + 2], w[8 * j + 3]);
          e4m3x4_to_bf16x4(v[j].z, w[8 * j + 4], w[8 * j + 5]);
          e4m3x4_to_bf16x4(v[j].w, w[8 * j + 6], w[8 * j + 7]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[slot], ph ^ 1, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        tc_fence_after();
        tmem_st32_wait(tl + slot * 64, w);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[slot]);
      }
      if (!ok) break;
      gs += nS;
    }
  } else if (warp < kTcXWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int frow = 32 * q + lane;
    const uint32_t tl = tbase + ((32u * q) << 16);
    uint16_t* stage = reinterpret_cast<uint16_t*>(se + (warp - 2 - kTcConvWarps) * (2 * 32 * 32 * 2));
    const int eh = (warp - 2 - kTcConvWarps) >> 2;  // which 32-token blocks: parity eh
    int eb = 0, ti = 0;
    uint32_t accph = 0, tph = 0;
    for (;;) {
      if (!__all_sync(0xffffffffu, mbar_wait(&tile_full[ti], tph, p.watch, kErrTimeoutEpilogue))) break;
      const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&tile_empty[ti]);
      if (++ti == kTcTileRing) { ti = 0; tph ^= 1; }
      if (T < 0) break;
      int f0, t0;
      tc_tile_coords(T, p.n_ftiles, p.n_ttiles, bt, f0, t0);
      const int valid = min(bt, p.M - t0);
      const int f = f0 + frow;
      const float s = f < p.N ? p.scale[f] : 0.f;
      const float b = (p.bias != nullptr && f < p.N) ? bf16_bits_to_float(p.bias[f]) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, accph, p.watch, kErrTimeoutEpilogue))) break;
      tc_fence_after();
      const bool store_rows = f0 + 32 * q < p.N;
      for (int c = 32 * eh; c < valid; c += 64) {
        uint32_t v[32];
        tmem_ld32_wait(tl + c, v);
        if (lane == 0) tma_store_wait_read<1>();
        __syncwarp();
        uint16_t* st = stage + eb * (32 * 32);
#pragma unroll
        for (int i = 0; i < 32; ++i) st[i * 32 + lane] = to_bf16_bits(epi_act<kAct>(fmaf(s, __uint_as_float(v[i]), b)));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (store_rows) tma_store_2d(&p.tm_y, st, f0 + 32 * q, t0 + c);
          tma_store_commit();
        }
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
    tmem_dealloc(tbase, 512);
  }
}

// Set-time preparation of the folded low-rank factor: A' = A / s_eff[n]
// split into a bf16 pair (hi = bf16(A'), lo = bf16(A' - hi)).  Flags any
// value whose pair would leave bf16's normal range.
__global__ void ll_fold_prep_kernel(const uint16_t* __restrict__ A, const float* __restrict__ s_eff,
                                    uint16_t* __restrict__ ahi, uint16_t* __restrict__ alo, int N, int r_pad,
                                    int* __restrict__ bad) {
  const size_t total = static_cast<size_t>(N) * r_pad;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / r_pad);
    const float a = bf16_bits_to_float(A[i]);
    const float ap = a / s_eff[n];
    const uint16_t h = to_bf16_bits(ap);
    const uint16_t l = to_bf16_bits(ap - bf16_bits_to_float(h));
    ahi[i] = h;
    alo[i] = l;
    const float m = fabsf(ap);
    if (!(m <= 0x1p100f) || (m != 0.f && m < 0x1p-100f)) atomicOr(bad, 1);
  }
}

// Copy of Q with the rows whose scale is zero cleared.
__global__ void ll_zero_rows_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scale,
                                    uint8_t* __restrict__ out, int N, int K) {
  const size_t total = static_cast<size_t>(N) * K;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / K);
    out[i] = scale[n] == 0.f ? 0 : q[i];
  }
}

}  // namespace llk
