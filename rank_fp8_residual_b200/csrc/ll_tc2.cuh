// CTA-pair fused kernel (sm_100a, tcgen05 cta_group::2) of the LiteLinear
// forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// evaluated per output row n as  y = s[n] * (Q x + A' t) + bias[n]  with
// A' = A / s[n] carried as a bf16 pair and t = x B^T carried as a bf16
// pair, exactly as in ll_tc.cuh (see the precision note there).
//
// Two CTAs of a cluster form one MMA of M = 256 output features: each CTA
// widens its own 128 residual rows into its own TMEM stages (its half of
// the A operand) and stages half of the token tile (its half of the B
// operand) in its own shared memory.  So every SM stages 128 Q rows and
// half of the x tile per K step, where the one-CTA kernel stages the whole
// x tile; each tensor core still reads the whole B operand, half of it from
// the peer.  Measured, a stage of eight MMAs takes about as long as in the
// one-CTA kernel at N = 224 and 256.  The accumulator of each CTA holds its
// 128 features x up to 256 tokens.
//
// The leader CTA (rank 0) issues the MMAs.  Its stage barrier a_full[s]
// collects, for each stage of two K steps: its eight converter arrivals,
// one arrival relayed from the peer's converters, and the leader x
// producer's arrival with the transaction bytes of both CTAs' x chunks
// (both CTAs' TMA loads complete on it).  MMA completion is committed to
// both CTAs.  The low-rank chunks (A'_hi, A'_lo, t_hi, t_lo) go through
// four ring slots each completing on a leader barrier of that slot.
//
// Work split: tiles of 256 features x bt tokens (bt a multiple of 32 up to
// 256, chosen per call) taken by the clusters from a device-wide counter
// in a grouped raster order.  The leader's scheduler warp takes each tile
// and writes it into the tile slot of both CTAs; the peer's scheduler warp
// tells the leader when all of the peer's roles have read a slot.
//
// Warp roles (28 warps per CTA): 0 TMA producer of Q, 1 MMA issuer (leader)
// or relay (peer) and TMEM allocator, 2-17 converters in two teams of eight
// on alternate stages (lane quadrant w%4, K step parity within a stage),
// 18-25 epilogue (two warps per lane quadrant on alternate 32-token
// blocks), 26 TMA producer of x and of the low-rank chunks, 27 tile
// scheduler (leader) or slot-release forwarder (peer).
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

struct Tc2Params {
  CUtensorMap tm_x;    // bf16 x: 3-D {64, M, K/64} box {64, bt/2, 2}, or 2-D [M, K] box {64, bt/2}; 128B swizzle
  CUtensorMap tm_q;    // u8 Q:   3-D {64, N, K/64} box {64, 128, 2}, or 2-D [N, K] box {64, 128}; 64B swizzle
  CUtensorMap tm_ahi;  // bf16 [N, r_pad]   box {klr, 128}, 128B (klr 64) / 64B (klr 32)
  CUtensorMap tm_alo;
  CUtensorMap tm_thi;  // bf16 [M, r_pad]   box {klr, bt/2}
  CUtensorMap tm_tlo;
  CUtensorMap tm_y;    // bf16 [M, N]       box {32, 32}
  const float* scale;    // effective per-row scale [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  int M, N, K, r_pad, klr;
  int dims3;     // 1: one 3-D load per stage for x and for Q; 0: two 2-D loads each
  int bt;        // tokens per tile (multiple of 32, <= 256); each CTA stages bt / 2 of them
  int n_fpairs;  // ceil(N / 256)
  int n_ttiles;  // ceil(M / bt)
  int* sched;    // [2]: tile counter, finished-leader counter (0 between launches)
  int lr_from_primary;
  int withhold;
  Watch watch;
};

constexpr int kT2ConvWarps = 16;
constexpr int kT2EpiWarps = 8;
constexpr int kT2XWarp = 2 + kT2ConvWarps + kT2EpiWarps;
constexpr int kT2SchedWarp = kT2XWarp + 1;
constexpr int kT2Threads = 32 * (kT2SchedWarp + 1);
constexpr int kT2TileRing = 2;
constexpr int kT2Group = 8;                   // token tiles per raster group
// Roles of a CTA that read each tile: Q producer, MMA / relay, converters,
// epilogue, x producer.
constexpr int kT2TileUsers = 1 + 1 + kT2ConvWarps + kT2EpiWarps + 1;
constexpr int kT2XUnit = 128 * kBK * 2;       // 16 KB: one CTA's 128 rows of one 64-wide bf16 chunk
constexpr int kT2SX = 8;                      // x ring slots (two per stage; low-rank chunks one each)
constexpr int kT2QChunk = 128 * kBK;          // 8 KB: 128 rows of one 64-wide e4m3 chunk
constexpr int kT2QSlot = 2 * kT2QChunk;       // one stage
constexpr int kT2SQ = 4;
constexpr int kT2NA = 4;                      // widened-Q stages in TMEM (two K steps, 64 columns)
constexpr int kT2Epi = kT2EpiWarps * 2 * 32 * 32 * 2;
constexpr int kT2ColA = 256;
static_assert(kT2SQ == kT2NA, "Q slots and TMEM stages advance together");
static_assert(kT2SX % 2 == 0, "the two x chunks of a stage take adjacent slots");

__host__ __device__ constexpr int tc2_smem_bytes() {
  return kT2SX * kT2XUnit + kT2SQ * kT2QSlot + kT2Epi + 1024 + 512;
}

// Feature pair and first token of tile T in the grouped raster order.
__device__ __forceinline__ void t2_tile_coords(const Tc2Params& p, int T, int& fp, int& t0) {
  const int per_group = kT2Group * p.n_fpairs;
  const int g = T / per_group;
  const int first_tt = g * kT2Group;
  const int gsize = min(kT2Group, p.n_ttiles - first_tt);
  const int idx = T - g * per_group;
  fp = idx / gsize;
  t0 = (first_tt + idx % gsize) * p.bt;
}

// Tokens each CTA of the pair stages for a tile (half of the MMA's N).
__device__ __forceinline__ int t2_half(const Tc2Params& p, int t0) {
  const int valid = min(p.bt, p.M - t0);
  return ((valid + 31) & ~31) >> 1;
}

// Reads the next tile from this CTA's tile ring (-1: no more tiles).
struct TileRing {
  int ti = 0;
  uint32_t tph = 0;
  __device__ bool next(uint64_t* tile_full, uint64_t* tile_empty, int* tile_slot, const Watch& w, int code,
                       bool whole_warp, int& T) {
    bool got = mbar_wait_cl(&tile_full[ti], tph, w, code);
    if (whole_warp) got = __all_sync(0xffffffffu, got);
    if (!got) return false;
    T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
    if (whole_warp) __syncwarp();
    if (!whole_warp || (threadIdx.x & 31) == 0) mbar_arrive(&tile_empty[ti]);
    if (++ti == kT2TileRing) { ti = 0; tph ^= 1; }
    return T >= 0;
  }
};

template <int kAct>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT2Threads, 1)
    ll_tc2_kernel(const __grid_constant__ Tc2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sx = smem;
  uint8_t* sq = sx + kT2SX * kT2XUnit;
  uint8_t* se = sq + kT2SQ * kT2QSlot;
  uint64_t* x_empty = reinterpret_cast<uint64_t*>(se + kT2Epi);  // both: MMA done with slot
  uint64_t* lr_full = x_empty + kT2SX;                            // leader: low-rank chunk landed
  uint64_t* q_full = lr_full + kT2SX;                             // local
  uint64_t* q_empty = q_full + kT2SQ;                             // local
  uint64_t* a_full = q_empty + kT2SQ;                             // leader: stage ready
  uint64_t* a_loc = a_full + kT2NA;                               // peer: its converters
  uint64_t* a_empty = a_loc + kT2NA;                              // both
  uint64_t* acc_full = a_empty + kT2NA;                           // both
  uint64_t* acc_empty = acc_full + 1;                             // leader: both CTAs' epilogues
  uint64_t* drain = acc_empty + 1;                                // leader
  uint64_t* tile_full = drain + 1;                                // both: the leader filled the slot
  uint64_t* tile_empty = tile_full + kT2TileRing;                 // both: local readers (+ peer's, leader)
  int* tile_slot = reinterpret_cast<int*>(tile_empty + kT2TileRing);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_slot + kT2TileRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int nK = (p.K + kBK - 1) / kBK;
  const int n_tiles = p.n_fpairs * p.n_ttiles;
  const int nS = (nK + 1) / 2;  // stages of two K steps (a step past K loads as zeros)
  const int klr = p.klr;
  const int nR = p.r_pad / klr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kT2SX; ++s) {
      mbar_init(&x_empty[s], 1);
      mbar_init(&lr_full[s], 1);
    }
    for (int s = 0; s < kT2SQ; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], kT2ConvWarps / 2);
    }
    for (int s = 0; s < kT2NA; ++s) {
      mbar_init(&a_full[s], kT2ConvWarps / 2 + 2);  // team + peer relay + x producer
      mbar_init(&a_loc[s], kT2ConvWarps / 2);
      mbar_init(&a_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kT2EpiWarps);
    mbar_init(drain, 1);
    for (int s = 0; s < kT2TileRing; ++s) {
      mbar_init(&tile_full[s], 1);
      mbar_init(&tile_empty[s], kT2TileUsers + (leader ? 1 : 0));
    }
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
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int hb = p.bt / 2;  // token rows of one CTA's x and t boxes

  if (warp == 0) {
    // ------------------------------------------------ TMA: this CTA's Q rows
    if (lane == 0 && !p.withhold) {
      int qi = 0;
      uint32_t qph = 0;
      long long nq = 0;
      bool ok = true;
      TileRing tr;
      int T;
      while (ok && tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutProducer, false, T)) {
        int fp, tok;
        t2_tile_coords(p, T, fp, tok);
        const int f0 = fp * 256 + 128 * static_cast<int>(rank);
        for (int s = 0; s < nS; ++s) {
          if (!mbar_wait(&q_empty[qi], qph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          uint8_t* dst = sq + qi * kT2QSlot;
          mbar_arrive_expect_tx(&q_full[qi], kT2QSlot);
          if (p.dims3) {
            tma_load_3d(dst, &p.tm_q, &q_full[qi], 0, f0, 2 * s);
          } else {
            tma_load_2d(dst, &p.tm_q, &q_full[qi], 2 * s * kBK, f0);
            tma_load_2d(dst + kT2QChunk, &p.tm_q, &q_full[qi], (2 * s + 1) * kBK, f0);
          }
          ++nq;
          if (++qi == kT2SQ) { qi = 0; qph ^= 1; }
        }
      }
      if (!ok) {
        for (long long i = (nq > kT2SQ ? nq - kT2SQ : 0); i < nq; ++i)
          mbar_wait_drain(&q_full[i % kT2SQ], static_cast<uint32_t>((i / kT2SQ) & 1), p.watch);
      }
    }
  } else if (warp == kT2XWarp) {
    // ----------------------- TMA: this CTA's x half, then low-rank chunks
    // The two x chunks of a stage sit back to back (the second hb rows of
    // 128 bytes after the first) in a pair of adjacent ring slots.
    if (lane == 0 && !p.withhold) {
      int xi = 0;
      uint32_t xph = 0;
      long long gsx = 0;  // stages issued
      bool issued = false, ok = true, waited_primary = false;
      const uint32_t x_bytes = 2u * 2u * hb * kBK * 2u;         // both CTAs, two chunks
      const uint32_t a_bytes = 2u * 128u * klr * 2u;            // both CTAs' A' chunk
      const uint32_t t_bytes = 2u * static_cast<uint32_t>(hb) * klr * 2u;  // both CTAs' t chunk
      TileRing tr;
      int T;
      while (ok && tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutProducer, false, T)) {
        int fp, tok;
        t2_tile_coords(p, T, fp, tok);
        const int half = t2_half(p, tok);
        const int f0 = fp * 256 + 128 * static_cast<int>(rank);
        const int t0 = tok + static_cast<int>(rank) * half;
        for (int s = 0; s < nS; ++s) {
          const int sa = xi;  // two adjacent slots: sa, sa + 1
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            if (++xi == kT2SX) { xi = 0; xph ^= 1; }
          }
          if (!ok) break;
          const int as = static_cast<int>(gsx % kT2NA);
          if (leader) mbar_arrive_expect_tx(&a_full[as], x_bytes);
          const uint32_t bar = mapa_shared(smem_u32(&a_full[as]), 0);
          uint8_t* dst = sx + sa * kT2XUnit;
          if (p.dims3) {
            tma_load_3d_pair(dst, &p.tm_x, bar, 0, t0, 2 * s);
          } else {
            tma_load_2d_pair(dst, &p.tm_x, bar, 2 * s * kBK, t0);
            tma_load_2d_pair(dst + hb * 128, &p.tm_x, bar, (2 * s + 1) * kBK, t0);
          }
          issued = true;
          ++gsx;
        }
        if (ok && nR > 0 && !waited_primary && p.lr_from_primary) {
          pdl_wait_primary();
          waited_primary = true;
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          const CUtensorMap* maps[4] = {&p.tm_ahi, &p.tm_alo, &p.tm_thi, &p.tm_tlo};
          const int rows[4] = {f0, f0, t0, t0};
          for (int li = 0; li < 4; ++li) {
            if (!mbar_wait(&x_empty[xi], xph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(&lr_full[xi], li < 2 ? a_bytes : t_bytes);
            tma_load_2d_pair(sx + xi * kT2XUnit, maps[li], mapa_shared(smem_u32(&lr_full[xi]), 0), jb * klr,
                             rows[li]);
            issued = true;
            if (++xi == kT2SX) { xi = 0; xph ^= 1; }
          }
        }
      }
      if (!ok && issued) {
        // Loads already issued must land before the CTA exits; they
        // complete on leader barriers that also count arrivals which may
        // never come now, so wait a bounded settle time (far above any load
        // latency); the final cluster barrier keeps both CTAs resident.
        const uint64_t c0 = clock_cycles();
        while (clock_cycles() - c0 < 400000ull) {  // >= 200 us at any clock up to 2 GHz
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------- MMA (leader only)
      int xi = 0, ai = 0;
      uint32_t aph = 0, accph = 0;
      uint32_t lr_ph = 0;  // per-slot phase bits of lr_full
      bool ok = true;
      TileRing tr;
      int T;
      while (ok && tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutMma, false, T)) {
        int fp, tok;
        t2_tile_coords(p, T, fp, tok);
        const uint32_t idesc = idesc_bf16(256, 2 * t2_half(p, tok));
        if (!mbar_wait_cl(acc_empty, accph ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        for (int s = 0; s < nS; ++s) {
          // One wait per stage: both CTAs' converted Q and x chunks.
          if (!mbar_wait_cl(&a_full[ai], aph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xb = smem_u32(sx + xi * kT2XUnit);
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const uint64_t bd = sdesc_kmajor_sw128(xb + sub * hb * 128);
            const uint32_t at = tbase + kT2ColA + ai * 64 + sub * 32;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_ts_pair(tbase, at + kk * 8, bd + 2 * kk, idesc, (s | sub | kk) != 0 ? 1u : 0u);
          }
          // Both chunks may sit in the first slot, so both slots are
          // released once the stage's MMAs are done.
          tc_commit_pair(&x_empty[xi], 0x3);
          tc_commit_pair(&x_empty[xi + 1], 0x3);
          xi = (xi + 2) % kT2SX;
          tc_commit_pair(&a_empty[ai], 0x3);
          if (++ai == kT2NA) { ai = 0; aph ^= 1; }
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          uint64_t d[4];
          int slots[4];
          for (int li = 0; li < 4; ++li) {
            if (!mbar_wait_cl(&lr_full[xi], (lr_ph >> xi) & 1u, p.watch, kErrTimeoutMma)) { ok = false; break; }
            lr_ph ^= 1u << xi;
            slots[li] = xi;
            const uint32_t sa = smem_u32(sx + xi * kT2XUnit);
            d[li] = klr == 64 ? sdesc_kmajor_sw128(sa) : sdesc_kmajor_sw64(sa);
            if (++xi == kT2SX) xi = 0;
          }
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < klr / 16; ++kk) {
            mma_ss_pair(tbase, d[0] + 2 * kk, d[2] + 2 * kk, idesc, 1u);  // A'_hi t_hi
            mma_ss_pair(tbase, d[0] + 2 * kk, d[3] + 2 * kk, idesc, 1u);  // A'_hi t_lo
            mma_ss_pair(tbase, d[1] + 2 * kk, d[2] + 2 * kk, idesc, 1u);  // A'_lo t_hi
          }
          for (int w = 0; w < 4; ++w) tc_commit_pair(&x_empty[slots[w]], 0x3);
        }
        if (!ok) break;
        tc_commit_pair(acc_full, 0x3);
        accph ^= 1;
      }
      // No MMA may still run when TMEM is released.
      tc_commit_pair(drain, 0x1);
      mbar_wait_drain(drain, 0, p.watch);
    } else if (lane == 0) {
      // ------------------------------------------------------ relay (peer)
      // One cross-CTA arrival per stage passes this CTA's "widened-Q stage
      // is in TMEM" on to the leader's stage barrier.
      const uint32_t a_full_leader = mapa_shared(smem_u32(&a_full[0]), 0);
      bool ok = true;
      long long g = 0;
      TileRing tr;
      int T;
      while (ok && tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutConvert, false, T)) {
        for (int s = 0; s < nS; ++s, ++g) {
          const int as = static_cast<int>(g % kT2NA);
          if (!mbar_wait(&a_loc[as], static_cast<uint32_t>((g / kT2NA) & 1), p.watch, kErrTimeoutConvert)) {
            ok = false;
            break;
          }
          mbar_arrive_cluster(a_full_leader + 8u * as);
        }
      }
    }
  } else if (warp < 2 + kT2ConvWarps) {
    // ----------------------------------------- e4m3 -> bf16 into TMEM stages
    // Stages are numbered across this CTA's tiles (g); team t takes the
    // stages g = t (mod 2).  Within a team, warp (q, par) widens K step
    // 2s + par of the stage for the rows of lane quadrant q: one full
    // 64-code row chunk per lane.  Stage g uses Q slot and TMEM stage
    // g mod 4, in phase (g / 4) mod 2.
    const int cw = warp - 2;
    const int team = cw >> 3;
    const int q = warp & 3;
    const int par = (cw >> 2) & 1;
    const int row = 32 * q + lane;
    const int sw = (row >> 1) & 3;
    const uint32_t tl = tbase + ((32u * q) << 16) + kT2ColA + 32 * par;
    uint64_t* a_arrive = leader ? a_full : a_loc;  // both local
    long long gs = 0;
    bool ok = true;
    TileRing tr;
    int T;
    while (ok && tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutConvert, true, T)) {
      for (long long g = gs + ((team - gs) & 1); g < gs + nS; g += 2) {
        const int slot = static_cast<int>(g % kT2SQ);
        const uint32_t ph = static_cast<uint32_t>((g / kT2SQ) & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&q_full[slot], ph, p.watch, kErrTimeoutConvert))) { ok = false; break; }
        uint4 v[4];
        const uint8_t* rb = sq + slot * kT2QSlot + par * kT2QChunk + row * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(rb + 16 * (j ^ sw));
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[slot]);
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e4m3x4_to_bf16x4(v[j].x, w[8 * j + 0], w[8 * j + 1]);
          e4m3x4_to_bf16x4(v[j].y, w[8 * j + 2], w[8 * j + 3]);
          e4m3x4_to_bf16x4(v[j].z, w[8 * j + 4], w[8 * j + 5]);
          e4m3x4_to_bf16x4(v[j].w, w[8 * j + 6], w[8 * j + 7]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[slot], ph ^ 1, p.watch, kErrTimeoutConvert))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32_wait(tl + slot * 64, w);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_arrive[slot]);
      }
      gs += nS;
    }
  } else if (warp < kT2XWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int frow = 32 * q + lane;
    const int eh = (warp - 2 - kT2ConvWarps) >> 2;  // which 32-token blocks: parity eh
    const uint32_t tl = tbase + ((32u * q) << 16);
    uint16_t* stage = reinterpret_cast<uint16_t*>(se + (warp - 2 - kT2ConvWarps) * (2 * 32 * 32 * 2));
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    int eb = 0;
    uint32_t accph = 0;
    TileRing tr;
    int T;
    while (tr.next(tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutEpilogue, true, T)) {
      int fp, tok;
      t2_tile_coords(p, T, fp, tok);
      const int valid = min(p.bt, p.M - tok);
      const int f0 = fp * 256 + 128 * static_cast<int>(rank);
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
          if (store_rows) tma_store_2d(&p.tm_y, st, f0 + 32 * q, tok + c);
          tma_store_commit();
        }
        eb ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(acc_empty);
        else
          mbar_arrive_cluster(acc_empty_leader);
      }
      accph ^= 1;
    }
    if (lane == 0) tma_store_wait<0>();
  } else if (warp == kT2SchedWarp && lane == 0) {
    if (leader) {
      // ----------------------------------------- tile scheduler (leader)
      // Each slot is refilled once this CTA's readers and the peer's
      // forwarder have released it; the tile number goes into both CTAs'
      // slots, the peer's by a cluster store ordered before the release
      // arrival on the peer's barrier.
      const uint32_t peer_slot = mapa_shared(smem_u32(&tile_slot[0]), 1);
      const uint32_t peer_full = mapa_shared(smem_u32(&tile_full[0]), 1);
      int ti = 0;
      uint32_t tph = 0;
      for (;;) {
        if (!mbar_wait_cl(&tile_empty[ti], tph ^ 1, p.watch, kErrTimeoutProducer)) break;
        const int got = atomicAdd(&p.sched[0], 1);
        const int T = got < n_tiles ? got : -1;
        *reinterpret_cast<volatile int*>(&tile_slot[ti]) = T;
        st_shared_cluster_u32(peer_slot + 4u * ti, static_cast<uint32_t>(T));
        mbar_arrive_cluster_release(peer_full + 8u * ti);
        mbar_arrive(&tile_full[ti]);
        if (++ti == kT2TileRing) { ti = 0; tph ^= 1; }
        if (T < 0) break;
      }
      // The last leader to finish resets the scheduler for the next launch.
      __threadfence();
      if (atomicAdd(&p.sched[1], 1) == static_cast<int>(gridDim.x / 2) - 1) {
        atomicExch(&p.sched[0], 0);
        atomicExch(&p.sched[1], 0);
      }
    } else {
      // ---------------------------------------- slot-release forwarder (peer)
      const uint32_t leader_empty = mapa_shared(smem_u32(&tile_empty[0]), 0);
      int ti = 0;
      uint32_t tph = 0;
      for (;;) {
        if (!mbar_wait_cl(&tile_full[ti], tph, p.watch, kErrTimeoutProducer)) break;
        const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
        if (T < 0) break;  // the last slot: nothing refills it
        if (!mbar_wait_cl(&tile_empty[ti], tph, p.watch, kErrTimeoutProducer)) break;
        mbar_arrive_cluster_release(leader_empty + 8u * ti);
        if (++ti == kT2TileRing) { ti = 0; tph ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs and epilogues are done with both TMEMs
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace llk
