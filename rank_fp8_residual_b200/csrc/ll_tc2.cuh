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
// widens its own 128 residual rows into its own TMEM stages (the A operand
// of the pair MMA) and stages half of the token tile (the B operand) in
// its own shared memory, so every SM reads 128 Q rows and half of the x
// tile per K step.  The accumulator of each CTA holds its 128 features x
// up to 256 tokens.  The leader CTA (rank 0) issues the MMAs; its
// barriers collect the TMA completions and the converter / epilogue
// arrivals of both CTAs, and MMA completion is committed to both CTAs.
//
// Work split: the (feature pair, token) rows of the layer are cut into
// one contiguous run per cluster, equal to within 32 tokens, and each run
// into pieces of at most 256 tokens (multiples of 32, so no two clusters
// write the same output rows).
//
// Warp roles (14 warps per CTA): 0 TMA producer, 1 MMA issuer (leader) and
// TMEM allocator, 2-9 converters (lane quadrant w%4, K half (w-2)/4),
// 10-13 epilogue.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

struct Tc2Params {
  CUtensorMap tm_x;    // bf16 x: 3-D {64, M, K/64} box {64, 128, xc} or 2-D [M, K] box {64, 128}; 128B swizzle
  CUtensorMap tm_q;    // u8 Q:   3-D {64, N, K/64} box {64, 128, qc} or 2-D [N, K] box {64, 128};  64B swizzle
  CUtensorMap tm_ahi;  // bf16 [N, r_pad]   box {klr, 128}, 128B (klr 64) / 64B (klr 32)
  CUtensorMap tm_alo;
  CUtensorMap tm_thi;  // bf16 [M, r_pad]   box {klr, 128}
  CUtensorMap tm_tlo;
  CUtensorMap tm_y;    // bf16 [M, N]       box {32, 32}
  const float* scale;    // effective per-row scale [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  int M, N, K, r_pad, klr;
  int dims3;     // 1: tm_x / tm_q are the 3-D views (K % 64 == 0)
  int xc, qc;    // 64-wide K chunks per x / Q load (1 or 2 / 1 or 4)
  int n_fpairs;  // ceil(N / 256)
  int m32;       // M rounded up to 32
  int seg;       // token rows per cluster (multiple of 32)
  int lr_from_primary;
  int withhold;
  Watch watch;
};

constexpr int kT2Threads = 448;
constexpr int kT2XRing = 128 * 1024;          // x / A' / t ring (slots of xc x 16 KB)
constexpr int kT2QRing = 64 * 1024;           // Q ring (slots of qc x 8 KB)
constexpr int kT2XUnit = 128 * kBK * 2;       // 16 KB: one CTA's 128 rows of one 64-wide bf16 chunk
constexpr int kT2QUnit = 128 * kBK;           // 8 KB: 128 rows of one 64-wide e4m3 chunk
constexpr int kT2MaxSlots = 8;
constexpr int kT2NA = 8;                      // widened-Q stages in TMEM
constexpr int kT2Epi = 4 * 2 * 32 * 32 * 2;   // 16384
constexpr int kT2ConvWarps = 8;
constexpr int kT2EpiWarps = 4;
constexpr int kT2ColA = 256;

__host__ __device__ constexpr int tc2_smem_bytes() { return kT2XRing + kT2QRing + kT2Epi + 1024 + 512; }

// The pieces of one cluster's run, in order.
struct PieceIter {
  int u, u_end, m32;
  __device__ PieceIter(const Tc2Params& p, int cid) {
    m32 = p.m32;
    const int total = p.n_fpairs * p.m32;
    u = min(total, cid * p.seg);
    u_end = min(total, u + p.seg);
  }
  // Returns false when the run is exhausted.
  __device__ bool next(int& fp, int& tok, int& len) {
    if (u >= u_end) return false;
    fp = u / m32;
    tok = u - fp * m32;
    len = min(256, min(m32 - tok, u_end - u));
    u += len;
    return true;
  }
};

struct Ring {
  int i = 0;
  uint32_t ph = 0;
  __device__ void adv(int n) {
    if (++i == n) { i = 0; ph ^= 1; }
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT2Threads, 1)
    ll_tc2_kernel(const __grid_constant__ Tc2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sx = smem;
  uint8_t* sq = sx + kT2XRing;
  uint8_t* se = sq + kT2QRing;
  uint64_t* x_full = reinterpret_cast<uint64_t*>(se + kT2Epi);  // leader: both CTAs' loads
  uint64_t* x_empty = x_full + kT2MaxSlots;                      // both: MMA done with slot
  uint64_t* q_full = x_empty + kT2MaxSlots;                      // local
  uint64_t* q_empty = q_full + kT2MaxSlots;                      // local
  uint64_t* a_full = q_empty + kT2MaxSlots;                      // leader: own warps + peer relay
  uint64_t* a_loc = a_full + kT2NA;                              // peer: its converter warps
  uint64_t* a_empty = a_loc + kT2NA;                             // both
  uint64_t* acc_full = a_empty + kT2NA;                          // both
  uint64_t* acc_empty = acc_full + 1;                            // leader: 8 epilogue warps
  uint64_t* drain = acc_empty + 1;                               // leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1;
  const int nK = (p.K + kBK - 1) / kBK;
  const int klr = p.klr;
  const int nR = p.r_pad / klr;
  const int xc = p.xc, qc = p.qc;
  const int xslot = xc * kT2XUnit, qslot = qc * kT2QUnit;
  const int nxs = kT2XRing / xslot, nqs = kT2QRing / qslot;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kT2MaxSlots; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], kT2ConvWarps);
    }
    for (int s = 0; s < kT2NA; ++s) {
      mbar_init(&a_full[s], kT2ConvWarps + 1);
      mbar_init(&a_loc[s], kT2ConvWarps);
      mbar_init(&a_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kT2EpiWarps);
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
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // --------------------------------------------------------------- TMA
    if (lane == 0 && !p.withhold) {
      Ring xr, qr;
      long long nq = 0;
      bool ok = true, waited_primary = false;
      const uint32_t a_box = 128u * klr * 2u;  // one CTA's A' or t chunk
      PieceIter it(p, cid);
      int fp, tok, len;
      while (ok && it.next(fp, tok, len)) {
        const int valid = min(len, p.M - tok);
        const int half = ((valid + 31) & ~31) >> 1;  // tokens per CTA in the MMA
        const int f0 = fp * 256 + 128 * static_cast<int>(rank);
        const int t0 = tok + static_cast<int>(rank) * half;
        for (int kb = 0; kb < nK && ok; ++kb) {
          if (kb % xc == 0) {
            if (!mbar_wait(&x_empty[xr.i], xr.ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(&x_full[xr.i], 2 * xslot);
            const uint32_t bar = mapa_shared(smem_u32(&x_full[xr.i]), 0);
            if (p.dims3)
              tma_load_3d_pair(sx + xr.i * xslot, &p.tm_x, bar, 0, t0, kb);
            else
              tma_load_2d_pair(sx + xr.i * xslot, &p.tm_x, bar, kb * kBK, t0);
            xr.adv(nxs);
          }
          if (kb % qc == 0) {
            if (!mbar_wait(&q_empty[qr.i], qr.ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
            mbar_arrive_expect_tx(&q_full[qr.i], qslot);
            if (p.dims3)
              tma_load_3d(sq + qr.i * qslot, &p.tm_q, &q_full[qr.i], 0, f0, kb);
            else
              tma_load_2d(sq + qr.i * qslot, &p.tm_q, &q_full[qr.i], kb * kBK, f0);
            ++nq;
            qr.adv(nqs);
          }
        }
        if (ok && nR > 0 && !waited_primary && p.lr_from_primary) {
          pdl_wait_primary();
          waited_primary = true;
        }
        // Low-rank chunks: loads A'_hi, A'_lo, t_hi, t_lo, packed xc per slot.
        for (int jb = 0; jb < nR && ok; ++jb) {
          const CUtensorMap* maps[4] = {&p.tm_ahi, &p.tm_alo, &p.tm_thi, &p.tm_tlo};
          const int rows[4] = {f0, f0, t0, t0};
          for (int li = 0; li < 4; ++li) {
            if (li % xc == 0) {
              if (!mbar_wait(&x_empty[xr.i], xr.ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
              if (leader) mbar_arrive_expect_tx(&x_full[xr.i], 2 * xc * a_box);
            }
            tma_load_2d_pair(sx + xr.i * xslot + (li % xc) * kT2XUnit, maps[li],
                             mapa_shared(smem_u32(&x_full[xr.i]), 0), jb * klr, rows[li]);
            if (li % xc == xc - 1) xr.adv(nxs);
          }
        }
      }
      if (!ok) {
        // Loads already issued must land before the CTA exits.  The local Q
        // ring is drained through its own barriers; the x slots of the peer
        // complete on the leader's barriers, so both CTAs also wait a
        // bounded settle time (far above any load latency) before the
        // teardown, and the final cluster barrier keeps both CTAs resident.
        for (long long i = (nq > nqs ? nq - nqs : 0); i < nq; ++i)
          mbar_wait_drain(&q_full[i % nqs], static_cast<uint32_t>((i / nqs) & 1), p.watch);
        const uint64_t t0 = clock_cycles();
        while (clock_cycles() - t0 < 400000ull) {  // >= 200 us at any clock up to 2 GHz
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- MMA (leader only)
    if (lane == 0 && leader) {
      Ring xr;
      int ai = 0;
      uint32_t aph = 0, accph = 0;
      bool ok = true;
      PieceIter it(p, cid);
      int fp, tok, len;
      while (ok && it.next(fp, tok, len)) {
        const int valid = min(len, p.M - tok);
        const int n_mma = (valid + 31) & ~31;
        const uint32_t idesc = idesc_bf16(256, n_mma);
        if (!mbar_wait_cl(acc_empty, accph ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        for (int kb = 0; kb < nK; ++kb) {
          const int sub = kb % xc;
          if (!mbar_wait_cl(&a_full[ai], aph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          if (sub == 0 && !mbar_wait_cl(&x_full[xr.i], xr.ph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sx + xr.i * xslot + sub * kT2XUnit));
          const uint32_t at = tbase + kT2ColA + ai * 32;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ts_pair(tbase, at + kk * 8, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair(&a_empty[ai], 0x3);
          if (++ai == kT2NA) { ai = 0; aph ^= 1; }
          if (sub == xc - 1 || kb == nK - 1) {
            tc_commit_pair(&x_empty[xr.i], 0x3);
            xr.adv(nxs);
          }
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          uint64_t d[4];
          int slots[4];
          int ns = 0;
          for (int li = 0; li < 4; ++li) {
            if (li % xc == 0) {
              if (!mbar_wait_cl(&x_full[xr.i], xr.ph, p.watch, kErrTimeoutMma)) { ok = false; break; }
              slots[ns++] = xr.i;
            }
            const uint32_t sa = smem_u32(sx + xr.i * xslot + (li % xc) * kT2XUnit);
            d[li] = klr == 64 ? sdesc_kmajor_sw128(sa) : sdesc_kmajor_sw64(sa);
            if (li % xc == xc - 1) xr.adv(nxs);
          }
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < klr / 16; ++kk) {
            mma_ss_pair(tbase, d[0] + 2 * kk, d[2] + 2 * kk, idesc, 1u);  // A'_hi t_hi
            mma_ss_pair(tbase, d[0] + 2 * kk, d[3] + 2 * kk, idesc, 1u);  // A'_hi t_lo
            mma_ss_pair(tbase, d[1] + 2 * kk, d[2] + 2 * kk, idesc, 1u);  // A'_lo t_hi
          }
          for (int w = 0; w < ns; ++w) tc_commit_pair(&x_empty[slots[w]], 0x3);
        }
        if (!ok) break;
        tc_commit_pair(acc_full, 0x3);
        accph ^= 1;
      }
      // No MMA may still run when TMEM is released.
      tc_commit_pair(drain, 0x1);
      mbar_wait_drain(drain, 0, p.watch);
    } else if (lane == 0) {
      // Peer: relay "this CTA's widened-Q stage is in TMEM" to the leader,
      // one cross-CTA arrival per stage.  The converter warps arrive
      // locally; the relay's wait and arrive pass their TMEM stores on to
      // the MMA issuer.
      const uint32_t a_full_leader = mapa_shared(smem_u32(&a_full[0]), 0);
      int ai = 0;
      uint32_t aph = 0;
      bool ok = true;
      PieceIter it(p, cid);
      int fp, tok, len;
      while (ok && it.next(fp, tok, len)) {
        for (int kb = 0; kb < nK; ++kb) {
          if (!mbar_wait(&a_loc[ai], aph, p.watch, kErrTimeoutConvert)) { ok = false; break; }
          mbar_arrive_cluster(a_full_leader + 8u * ai);
          if (++ai == kT2NA) { ai = 0; aph ^= 1; }
        }
      }
    }
  } else if (warp < 2 + kT2ConvWarps) {
    // ----------------------------------------- e4m3 -> bf16 into TMEM stages
    const int q = warp & 3;
    const int khalf = (warp - 2) >> 2;
    const int row = 32 * q + lane;
    const int sw = (row >> 1) & 3;
    const uint32_t tl = tbase + ((32u * q) << 16) + kT2ColA + 16 * khalf;
    uint64_t* a_arrive = leader ? a_full : a_loc;  // both local
    Ring qr;
    int ai = 0;
    uint32_t aph = 0;
    bool ok = true;
    PieceIter it(p, cid);
    int fp, tok, len;
    // Reads k-step kb of the piece from the Q ring (waiting for its slot
    // when kb starts one, releasing the slot after its last k-step).
    auto fetch = [&](int kb, uint4& v0, uint4& v1) -> bool {
      const int sub = kb % qc;
      if (sub == 0 &&
          !__all_sync(0xffffffffu, mbar_wait(&q_full[qr.i], qr.ph, p.watch, kErrTimeoutConvert)))
        return false;
      const uint8_t* rb = sq + qr.i * qslot + sub * kT2QUnit + row * 64;
      v0 = *reinterpret_cast<const uint4*>(rb + 16 * ((2 * khalf) ^ sw));
      v1 = *reinterpret_cast<const uint4*>(rb + 16 * ((2 * khalf + 1) ^ sw));
      if (sub == qc - 1 || kb == nK - 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[qr.i]);
        qr.adv(nqs);
      }
      return true;
    };
    while (ok && it.next(fp, tok, len)) {
      uint4 v0, v1;
      if (!fetch(0, v0, v1)) break;
      for (int kb = 0; kb < nK; ++kb) {
        uint32_t w[16];
        e4m3x4_to_bf16x4(v0.x, w[0], w[1]);
        e4m3x4_to_bf16x4(v0.y, w[2], w[3]);
        e4m3x4_to_bf16x4(v0.z, w[4], w[5]);
        e4m3x4_to_bf16x4(v0.w, w[6], w[7]);
        e4m3x4_to_bf16x4(v1.x, w[8], w[9]);
        e4m3x4_to_bf16x4(v1.y, w[10], w[11]);
        e4m3x4_to_bf16x4(v1.z, w[12], w[13]);
        e4m3x4_to_bf16x4(v1.w, w[14], w[15]);
        if (kb + 1 < nK && !fetch(kb + 1, v0, v1)) {
          ok = false;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[ai], aph ^ 1, p.watch, kErrTimeoutConvert))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(tl + ai * 32, w);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_arrive[ai]);
        if (++ai == kT2NA) { ai = 0; aph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int frow = 32 * q + lane;
    const uint32_t tl = tbase + ((32u * q) << 16);
    uint16_t* stage = reinterpret_cast<uint16_t*>(se + (warp - 2 - kT2ConvWarps) * (2 * 32 * 32 * 2));
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    int eb = 0;
    uint32_t accph = 0;
    PieceIter it(p, cid);
    int fp, tok, len;
    while (it.next(fp, tok, len)) {
      const int valid = min(len, p.M - tok);
      const int f0 = fp * 256 + 128 * static_cast<int>(rank);
      const int f = f0 + frow;
      const float s = f < p.N ? p.scale[f] : 0.f;
      const float b = (p.bias != nullptr && f < p.N) ? bf16_bits_to_float(p.bias[f]) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, accph, p.watch, kErrTimeoutEpilogue))) break;
      tc_fence_after();
      const bool store_rows = f0 + 32 * q < p.N;
      for (int c = 0; c < valid; c += 32) {
        uint32_t v[32];
        tmem_ld32_wait(tl + c, v);
        if (lane == 0) tma_store_wait_read<1>();
        __syncwarp();
        uint16_t* st = stage + eb * (32 * 32);
#pragma unroll
        for (int i = 0; i < 32; ++i) st[i * 32 + lane] = to_bf16_bits(fmaf(s, __uint_as_float(v[i]), b));
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
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs and epilogues are done with both TMEMs
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

// t = x B^T for r_pad <= 128 with warp-level MMA.  A block of four warps
// owns 16 tokens x 32 columns of t; the warps split K in quarters and
// their partial sums are added in warp order through shared memory (a
// fixed order, so results do not depend on timing).  Small enough (16 KB
// of shared memory, no TMEM) to run on the same SMs as the CTA-pair kernel
// while that one streams the residual GEMM.  Within each 32-wide K block,
// thread t of a quad owns the 8 consecutive K indices 8t .. 8t+7 of both
// operands (the dot product does not depend on the order of K, and both
// operands use the same assignment).
constexpr int kLrwUnroll = 4;
__global__ void __launch_bounds__(128) ll_lrdown_warp_kernel(const uint16_t* __restrict__ x,
                                                             const uint16_t* __restrict__ B,
                                                             uint16_t* __restrict__ t_hi,
                                                             uint16_t* __restrict__ t_lo, int M, int K, int r_pad) {
  __shared__ float red[4][16][33];
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int m0 = blockIdx.x * 16;
  const int j0 = blockIdx.y * 32;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = m0 + g, r1 = m0 + g + 8;
  const bool v0 = r0 < M, v1 = r1 < M;
  const uint16_t* x0 = x + static_cast<size_t>(v0 ? r0 : 0) * K;
  const uint16_t* x1 = x + static_cast<size_t>(v1 ? r1 : 0) * K;
  const uint16_t* bp[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) bp[b] = B + static_cast<size_t>(j0 + b * 8 + g) * K;
  // K quarter of this warp, in 32-wide blocks
  const int nkb = (K + 31) / 32;
  const int kb_lo = (nkb * warp) / 4, kb_hi = (nkb * (warp + 1)) / 4;
  float acc[4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int kb = kb_lo; kb < kb_hi; kb += kLrwUnroll) {
    uint4 a0[kLrwUnroll], a1[kLrwUnroll], bb[kLrwUnroll][4];
#pragma unroll
    for (int u = 0; u < kLrwUnroll; ++u) {
      const int kc = (kb + u) * 32 + 8 * t;
      const bool kin = (kb + u) < kb_hi && kc < K;  // K is a multiple of 16
      a0[u] = (v0 && kin) ? __ldg(reinterpret_cast<const uint4*>(x0 + kc)) : zero;
      a1[u] = (v1 && kin) ? __ldg(reinterpret_cast<const uint4*>(x1 + kc)) : zero;
#pragma unroll
      for (int b = 0; b < 4; ++b) bb[u][b] = kin ? __ldg(reinterpret_cast<const uint4*>(bp[b] + kc)) : zero;
    }
#pragma unroll
    for (int u = 0; u < kLrwUnroll; ++u) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        mma_m16n8k16_bf16(acc[b], a0[u].x, a1[u].x, a0[u].y, a1[u].y, bb[u][b].x, bb[u][b].y);
        mma_m16n8k16_bf16(acc[b], a0[u].z, a1[u].z, a0[u].w, a1[u].w, bb[u][b].z, bb[u][b].w);
      }
    }
  }
  // fragment -> shared: rows g, g+8; columns b*8 + 2t, +1
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    red[warp][g][b * 8 + 2 * t] = acc[b][0];
    red[warp][g][b * 8 + 2 * t + 1] = acc[b][1];
    red[warp][g + 8][b * 8 + 2 * t] = acc[b][2];
    red[warp][g + 8][b * 8 + 2 * t + 1] = acc[b][3];
  }
  __syncthreads();
  // 128 threads x 2 adjacent columns x 2 rows = 16 x 32 outputs
  const int row = threadIdx.x >> 4;        // 0..7, and row + 8
  const int col = (threadIdx.x & 15) * 2;  // 0..30
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int rr = row + 8 * h;
    const int m = m0 + rr;
    if (m >= M) continue;
    float e0 = 0.f, e1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      e0 += red[w][rr][col];
      e1 += red[w][rr][col + 1];
    }
    const uint16_t h0 = to_bf16_bits(e0), h1 = to_bf16_bits(e1);
    const uint32_t hv = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
    const uint32_t lv = pack_bf16x2(e0 - bf16_bits_to_float(h0), e1 - bf16_bits_to_float(h1));
    *reinterpret_cast<uint32_t*>(t_hi + static_cast<size_t>(m) * r_pad + j0 + col) = hv;
    *reinterpret_cast<uint32_t*>(t_lo + static_cast<size_t>(m) * r_pad + j0 + col) = lv;
  }
}

}  // namespace llk
