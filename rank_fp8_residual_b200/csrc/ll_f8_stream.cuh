// Small-M streaming kernel on FP8 operands (sm_100a) of the LiteLinear forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// for M <= 64 tokens, where the forward is bound by reading Q (N*K bytes)
// and A (2*N*r bytes) from HBM once.  The residual codes go from the TMA
// ring straight into tcgen05.mma kind::f8f6f4: x is split per token into
// two e4m3fn terms (ll_xsplit_kernel: x = 2^e_m (x_hi + x_lo), the split
// of ll_f8.cuh), so no warp widens Q and the tensor core reads it as the
// bytes that came from HBM.
//
//   acc_Q  [128 features x Mt tokens] += Q[128 x 32] * x_hi[Mt x 32]^T (+ x_lo)
//   acc_LR [128 x Mt]                 += A[128 x 16] * t'_hi[Mt x 16]^T (+ t'_lo)
//   y[m, n] = bf16( 2^e_m * (scale[n] * acc_Q + acc_LR) + bias[n] )
//
// with t' = t / 2^e_m written by ll_lrdown_kernel, which runs beside this
// grid on the SMs it leaves free (programmatic dependent launch; only the
// low-rank loads wait for it).
//
// Work split (stream-K over weight bytes).  A 128-feature tile is a row of
// units of 16 KB of weights: nS units of 128 residual codes per row, then
// nR units of 64 columns of A.  The n_ftiles * (nS + nR) units, tile-major,
// are cut into one equal contiguous range per CTA, so every CTA streams the
// same number of bytes whatever N, K and r are.  A range is cut at tile
// boundaries into segments, which a CTA processes last segment first: its
// last segment starts at a tile's first unit, so the low-rank units, which
// wait for t, come late in every CTA's stream.  A tile whose units fall in
// several ranges ("split tile") is finished by the last of its CTAs to
// arrive: the others leave fp32 partials of scale * acc_Q + acc_LR, and the
// finisher adds all of them in CTA order (a fixed order, whoever is last).
//
// Warp roles (8 warps): 0 TMA producer of the weight units (HBM), 1 and 7
// MMA issuers (even and odd units; warp 1 also allocates TMEM), 2 TMA
// producer of the activation units (x_hi / x_lo, or t'_hi / t'_lo, from
// L2), 3-6 epilogue (TMEM lanes 32 * (warp % 4) ...).
//
// Issue rate (measured on B200).  At M = 128 a tcgen05.mma costs ~45 cycles
// for N <= 32, 48 at N = 64, 64 at N = 128 and 128 at N = 256, for
// kind::f8f6f4 (K = 32) and kind::f16 (K = 16) alike, issued back to back:
// at small N the operand reads from shared memory (4 KB of A per MMA) set
// the pace.  A unit is 8 MMAs, ~450 cycles.  But any shared-memory access
// by the issuing thread, an mbarrier wait included, waits behind the
// operand reads of the MMAs it has issued, so one issuer waiting for each
// unit's data ran at ~850 cycles per unit.  Two issuers on alternate units
// keep the tensor core fed while the other waits: ~520 cycles per unit.
// Each issuer has its own accumulator pair (double-buffered in TMEM, so a
// segment's epilogue overlaps the next segment's MMAs); the epilogue adds
// the two in a fixed order.  The issue loop does no per-MMA arithmetic
// beyond adding constants to descriptors made once per unit.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

struct F8sParams {
  CUtensorMap tm_q;    // u8 Q [N, K]           box {128, 128}, 128B swizzle
  CUtensorMap tm_xh;   // u8 x_hi [M, K]        box {128, Mt},  128B swizzle
  CUtensorMap tm_xl;   // u8 x_lo [M, K]
  CUtensorMap tm_a;    // bf16 A [N, r_pad]     box {64, 128},  128B swizzle
  CUtensorMap tm_thi;  // bf16 t'_hi [M, r_pad] box {64, Mt},   128B swizzle
  CUtensorMap tm_tlo;  // bf16 t'_lo [M, r_pad]
  const int* e_tok;      // [M] token exponents
  const float* scale;    // [N]
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  uint16_t* y;           // [M, N] bf16 bits
  float* part;           // [2 * ctas][64][128] fp32 partials of split tiles
  int* cnt;              // [n_ftiles] arrivals on split tiles (0 between launches)
  int M, N, K, r_pad;
  int Mt;                // MMA N: tokens padded to a multiple of 16, 16..64
  int terms;             // 1: x_hi only (FP8 activations); 2: x_hi + x_lo
  int n_ftiles;
  int ctas;              // gridDim.x
  int w_stages;          // weight ring depth (16 KB slots)
  int lr_from_primary;   // 1: t' is written by the preceding kernel
  int withhold;          // debug: the producers issue nothing, so every consumer's wait runs out
  Watch watch;
};

constexpr int kSsThreads = 8 * 32;
constexpr int kSsMma2Warp = 7;
constexpr int kSsEpiWarp0 = 3;
constexpr int kSsWUnit = 16384;         // one weight unit: 128 rows x 128 bytes
constexpr int kSsMaxW = 12;             // weight slots at most
constexpr int kSsX = 4;                 // activation slots
constexpr int kSsMaxMt = 64;
constexpr int kSsPartFloats = kSsMaxMt * 128;  // one partial: [64 tokens][128 features]
constexpr int kSsRingBytes = 208 * 1024;

__host__ __device__ constexpr int ss_xslot_bytes(int Mt) { return 2 * Mt * 128; }
__host__ __device__ constexpr int ss_w_stages(int Mt) {
  return (kSsRingBytes - kSsX * ss_xslot_bytes(Mt)) / kSsWUnit < kSsMaxW
             ? (kSsRingBytes - kSsX * ss_xslot_bytes(Mt)) / kSsWUnit
             : kSsMaxW;
}
__host__ __device__ constexpr int ss_smem_bytes(int Mt) {
  return ss_w_stages(Mt) * kSsWUnit + kSsX * ss_xslot_bytes(Mt) + 1024 /*align*/ + 512 /*barriers*/;
}
__host__ __device__ constexpr int ss_smem_max() { return ss_smem_bytes(16) > ss_smem_bytes(64) ? ss_smem_bytes(16) : ss_smem_bytes(64); }

// The units of the grid and each CTA's share of them.
struct SsWork {
  int nS, nU, U, C;
  __device__ SsWork(const F8sParams& p) {
    nS = (p.K + 127) / 128;
    nU = nS + (p.r_pad + 63) / 64;
    U = p.n_ftiles * nU;
    C = p.ctas;
  }
  __device__ int begin(int c) const { return static_cast<int>(static_cast<long long>(U) * c / C); }
  // CTA that holds unit u.
  __device__ int owner(int u) const {
    int c = static_cast<int>(static_cast<long long>(u) * C / U);
    while (c + 1 < C && begin(c + 1) <= u) ++c;
    while (c > 0 && begin(c) > u) --c;
    return c;
  }
  // Partial slot of CTA j's segment on split tile f: 2j for its first
  // segment, 2j + 1 for its last when that is another one.
  __device__ int slot(int j, int f) const { return 2 * j + (begin(j) < f * nU ? 1 : 0); }
};

// This CTA's segments, last first: tile f and its units [a, b).
struct SsSegs {
  int u0, u1, nU, f, f_end;
  __device__ SsSegs(const SsWork& w, int c) : u0(w.begin(c)), u1(w.begin(c + 1)), nU(w.nU) {
    f = u1 > u0 ? (u1 - 1) / nU : -1;
    f_end = u1 > u0 ? u0 / nU : 0;
  }
  __device__ bool next(int& tile, int& a, int& b) {
    if (f < f_end) return false;
    tile = f;
    a = max(u0 - f * nU, 0);
    b = min(u1 - f * nU, nU);
    --f;
    return true;
  }
};

template <int kAct>
__global__ void __launch_bounds__(kSsThreads, 1) ll_f8_stream_kernel(const __grid_constant__ F8sParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int nW = p.w_stages;
  const int xsb = ss_xslot_bytes(p.Mt);
  uint8_t* wring = smem;
  uint8_t* xring = wring + nW * kSsWUnit;
  uint64_t* wfull = reinterpret_cast<uint64_t*>(xring + kSsX * xsb);
  uint64_t* wempty = wfull + kSsMaxW;
  uint64_t* xfull = wempty + kSsMaxW;
  uint64_t* xempty = xfull + kSsX;
  uint64_t* afull = xempty + kSsX;   // [2] accumulator buffer written
  uint64_t* aempty = afull + 2;      // [2] accumulator buffer read by the epilogue
  uint64_t* drain = aempty + 2;      // [2] one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  int* s_last = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = static_cast<int>(blockIdx.x);
  const SsWork wk(p);
  const int nS = wk.nS;
  const int Mt = p.Mt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int s = 0; s < kSsX; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 2);  // both issuers
      mbar_init(&aempty[b], 4);
      mbar_init(&drain[b], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_xh);
    if (p.terms == 2) tma_prefetch_desc(&p.tm_xl);
    if (p.r_pad > 0) {
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

  if (warp == 0 || warp == 2) {
    // ------------------------------------ TMA producers: weights / activations
    if (lane == 0) {
      const bool wside = warp == 0;
      const int ns = wside ? nW : kSsX;
      int slot = 0;
      uint32_t ph = 0;
      bool ok = !p.withhold, issued = false, waited = false;
      SsSegs sg(wk, c);
      int f, a, b;
      while (ok && sg.next(f, a, b)) {
        for (int u = a; u < b; ++u) {
          uint64_t* emp = wside ? &wempty[slot] : &xempty[slot];
          uint64_t* ful = wside ? &wfull[slot] : &xfull[slot];
          if (!mbar_wait(emp, ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          if (wside) {
            uint8_t* dst = wring + slot * kSsWUnit;
            mbar_arrive_expect_tx(ful, kSsWUnit);
            if (u < nS)
              tma_load_2d(dst, &p.tm_q, ful, u * 128, f * 128);
            else
              tma_load_2d(dst, &p.tm_a, ful, (u - nS) * 64, f * 128);
          } else {
            uint8_t* dst = xring + slot * xsb;
            if (u < nS) {
              mbar_arrive_expect_tx(ful, static_cast<uint32_t>(p.terms * Mt * 128));
              tma_load_2d(dst, &p.tm_xh, ful, u * 128, 0);
              if (p.terms == 2) tma_load_2d(dst + Mt * 128, &p.tm_xl, ful, u * 128, 0);
            } else {
              if (!waited && p.lr_from_primary) {
                pdl_wait_primary();
                waited = true;
              }
              mbar_arrive_expect_tx(ful, static_cast<uint32_t>(2 * Mt * 128));
              tma_load_2d(dst, &p.tm_thi, ful, (u - nS) * 64, 0);
              tma_load_2d(dst + Mt * 128, &p.tm_tlo, ful, (u - nS) * 64, 0);
            }
          }
          issued = true;
          if (++slot == ns) { slot = 0; ph ^= 1; }
        }
      }
      if (!ok && issued) {
        // Loads already issued must land before the CTA exits: wait a
        // bounded settle time far above any load latency.
        const uint64_t c0 = clock_cycles();
        while (clock_cycles() - c0 < 400000ull) {  // >= 200 us at any clock up to 2 GHz
        }
      }
    }
  } else if (warp == 1 || warp == kSsMma2Warp) {
    if (lane == 0) {
      // ------------------------------------------ MMA issuers (units k % 2)
      const int me = warp == 1 ? 0 : 1;
      const uint32_t id8 = idesc_e4m3(128, Mt);
      const uint32_t id16 = idesc_bf16(128, Mt);
      int ws = 0, xs = 0, seg = 0, kpar = 0;  // ring positions of the running unit k, and k % 2
      uint32_t wph = 0, xph = 0;
      bool ok = true;
      SsSegs sg(wk, c);
      int f, a, b;
      while (ok && sg.next(f, a, b)) {
        const int buf = seg & 1;
        if (!mbar_wait(&aempty[buf], ((seg >> 1) & 1) ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        // accumulator pair (buffer, issuer): columns 128 * (2 buf + me)
        const uint32_t dq = tbase + 128u * (2 * buf + me), dlr = dq + 64u;
        uint32_t qacc = 0, lracc = 0;  // 0 until an accumulator's first MMA of the segment
        for (int u = a; u < b; ++u) {
          if (kpar != me) {
            kpar ^= 1;
            if (++ws == nW) { ws = 0; wph ^= 1; }
            if (++xs == kSsX) { xs = 0; xph ^= 1; }
            continue;
          }
          kpar ^= 1;
          if (!mbar_wait(&wfull[ws], wph, p.watch, kErrTimeoutMma) ||
              !mbar_wait(&xfull[xs], xph, p.watch, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(wring + ws * kSsWUnit), xa = smem_u32(xring + xs * xsb);
          // Descriptors once per unit; a K step of 32 bytes adds 2 to the
          // encoded start address, the second x term Mt * 128 bytes.
          const uint64_t ad = sdesc_kmajor_sw128(wa), bd = sdesc_kmajor_sw128(xa);
          const uint64_t bd2 = bd + static_cast<uint64_t>(Mt * 8);
          if (u < nS) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f8(dq, ad + 2 * kk, bd + 2 * kk, id8, qacc);
              qacc = 1;
            }
            if (p.terms == 2) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) mma_f8(dq, ad + 2 * kk, bd2 + 2 * kk, id8, 1u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_ss(dlr, ad + 2 * kk, bd + 2 * kk, id16, lracc);
              lracc = 1;
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_ss(dlr, ad + 2 * kk, bd2 + 2 * kk, id16, 1u);
          }
          tc_commit(&wempty[ws]);
          tc_commit(&xempty[xs]);
          if (++ws == nW) { ws = 0; wph ^= 1; }
          if (++xs == kSsX) { xs = 0; xph ^= 1; }
        }
        if (!ok) break;
        tc_commit(&afull[buf]);
        ++seg;
      }
      // Every MMA this thread issued has completed before TMEM is freed.
      tc_commit(&drain[me]);
      mbar_wait_drain(&drain[me], 0, p.watch);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 3-6)
    const int q = warp & 3;
    const int row = 32 * q + lane;  // feature within the tile
    const uint32_t tl = tbase + ((32u * q) << 16);
    const int nch = Mt / 16;
    int seg = 0, k0 = 0;  // k0: the running unit number of the segment's first unit
    SsSegs sg(wk, c);
    int f, a, b;
    while (sg.next(f, a, b)) {
      const int buf = seg & 1;
      // Which issuer wrote which accumulator: the segment's residual units
      // are its units below nS, numbered k0, k0 + 1, ...; issuer k % 2.
      const int nq = max(0, min(b, nS) - a), nl = max(0, b - max(a, nS));
      const int kl = k0 + nq;  // number of the first low-rank unit
      const bool q0 = nq >= 2 || (nq == 1 && (k0 & 1) == 0), q1 = nq >= 2 || (nq == 1 && (k0 & 1) == 1);
      const bool l0 = nl >= 2 || (nl == 1 && (kl & 1) == 0), l1 = nl >= 2 || (nl == 1 && (kl & 1) == 1);
      k0 += b - a;
      // One decision for all four warps (they meet at named barriers below).
      const bool got = __all_sync(0xffffffffu, mbar_wait(&afull[buf], (seg >> 1) & 1, p.watch, kErrTimeoutEpilogue));
      if (!named_bar_and(1, 128, got)) break;
      tc_fence_after();
      const int n = f * 128 + row;
      const bool nin = n < p.N;
      const float sn = nin ? __ldg(p.scale + n) : 0.f;
      float v[kSsMaxMt];
#pragma unroll
      for (int m = 0; m < kSsMaxMt; ++m) v[m] = 0.f;
#pragma unroll
      for (int j = 0; j < kSsMaxMt / 16; ++j) {
        if (j < nch) {
          // issuer 0's pair at columns 256 buf, issuer 1's at 256 buf + 128
          const uint32_t t0 = tl + 256u * buf + 16u * j, t1 = t0 + 128u;
          uint32_t rq0[16], rl0[16], rq1[16], rl1[16];
          tmem_ld16x2_wait(t0, rq0, t0 + 64u, rl0);
          tmem_ld16x2_wait(t1, rq1, t1 + 64u, rl1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float sq = (q0 ? __uint_as_float(rq0[i]) : 0.f) + (q1 ? __uint_as_float(rq1[i]) : 0.f);
            const float sl = (l0 ? __uint_as_float(rl0[i]) : 0.f) + (l1 ? __uint_as_float(rl1[i]) : 0.f);
            v[16 * j + i] = fmaf(sn, sq, sl);
          }
        }
      }
      // The accumulator buffer is free for the segment after next.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[buf]);
      ++seg;

      bool finish = true;
      if (a > 0 || b < wk.nU) {
        // Split tile: leave this CTA's partial, count the arrival.
        const int c_first = wk.owner(f * wk.nU), c_last = wk.owner(f * wk.nU + wk.nU - 1);
        float* mine = p.part + static_cast<size_t>(wk.slot(c, f)) * kSsPartFloats;
#pragma unroll
        for (int j = 0; j < kSsMaxMt / 16; ++j)
          if (j < nch)
#pragma unroll
            for (int i = 0; i < 16; ++i) __stcg(mine + (16 * j + i) * 128 + row, v[16 * j + i]);
        __threadfence();
        named_bar_sync(1, 128);
        if (warp == kSsEpiWarp0 && lane == 0) {
          const int old = atomicAdd(p.cnt + f, 1);
          const bool last = old == c_last - c_first;
          if (last) p.cnt[f] = 0;  // every contributor has arrived: ready for the next launch
          *reinterpret_cast<volatile int*>(s_last) = last ? 1 : 0;
        }
        named_bar_sync(1, 128);
        finish = *reinterpret_cast<volatile int*>(s_last) != 0;
        named_bar_sync(1, 128);  // s_last is read by all before the next split tile writes it
        if (finish) {
          __threadfence();  // acquire: the other CTAs' partials are visible
          float tot[kSsMaxMt];
#pragma unroll
          for (int m = 0; m < kSsMaxMt; ++m) tot[m] = 0.f;
          for (int jc = c_first; jc <= c_last; ++jc) {
            if (jc == c) {
#pragma unroll
              for (int m = 0; m < kSsMaxMt; ++m) tot[m] += v[m];
              continue;
            }
            const float* src = p.part + static_cast<size_t>(wk.slot(jc, f)) * kSsPartFloats;
#pragma unroll
            for (int j = 0; j < kSsMaxMt / 16; ++j)
              if (j < nch)
#pragma unroll
                for (int i = 0; i < 16; ++i) tot[16 * j + i] += __ldcg(src + (16 * j + i) * 128 + row);
          }
#pragma unroll
          for (int m = 0; m < kSsMaxMt; ++m) v[m] = tot[m];
        }
      }
      if (finish && nin) {
        const float bn = p.bias != nullptr ? bf16_bits_to_float(p.bias[n]) : 0.f;
#pragma unroll
        for (int m = 0; m < kSsMaxMt; ++m)
          if (m < p.M && m < Mt)
            p.y[static_cast<size_t>(m) * p.N + n] =
                to_bf16_bits(epi_act<kAct>(fmaf(exp2_int(__ldg(p.e_tok + m)), v[m], bn)));
      }
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
