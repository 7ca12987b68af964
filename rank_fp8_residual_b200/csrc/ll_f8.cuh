// FP8-operand kernels (sm_100a) of the LiteLinear forward
//
//     y = (x B^T) A^T + scale * (x Q^T) + bias            (LiteLinear README,
//                                                          introduction)
//
// The residual product runs on tcgen05 kind::f8f6f4 with Q as stored
// (e4m3fn, README "Features") and x carried per token m as
//
//     x[m, k] ~= 2^e_m * (hi[m, k] + lo[m, k])        hi, lo e4m3fn codes
//
// where 2^e_m is the smallest power of two with max_k |x[m, k]| <= 448 * 2^e_m,
// hi is x / 2^e_m rounded to e4m3fn (nearest even) and lo the rounding of
// the remainder.  One term (hi only) is the FP8-activation variant; two
// terms reproduce x exactly wherever |x| >= 2^e_m / 4 and within
// 2^(e_m - 10) below that, which keeps the forward inside the accuracy
// bound of the bf16 path at the cost of one bf16 pass (an e4m3 MMA does
// twice the work of a bf16 one per cycle).  No operand is widened.
//
// With t' = t / 2^e_m (the down-projection divides by the token's power of
// two; exact) and A' = A / s[n] (the set-time bf16 pair of ll_tc.cuh):
//
//     y[m, n] = s[n] * 2^e_m * ( sum_k (hi + lo)[m, k] Q[n, k]
//                                + sum_j t'[m, j] A'[n, j] ) + bias[n]
//
// so one fp32 accumulator holds both terms; the low-rank part takes three
// bf16 MMAs per K step (t'_hi A'_hi + t'_lo A'_hi + t'_hi A'_lo).
//
// Kernel 1, ll_xsplit_kernel: one warp per token row; the row maximum,
// e_m, and the codes.  Kernel 2, ll_f8_kernel: persistent CTA pairs
// (cta_group::2).  A tile is 256 tokens x 256 features: each CTA stages
// its 128 token rows of hi (and lo) and its 128 feature rows of Q per 128-
// wide K step (16 KB each) and holds the accumulator of its 128 tokens x
// all 256 features in TMEM, double-buffered (2 x 256 columns), so the
// epilogue of one tile runs under the MMAs of the next.  Tokens are the
// MMA M side, so each thread of the epilogue owns one token row and stores
// contiguous features.
//
// Work split: data-parallel waves of tiles, then stream-K over the last
// (partial) wave, so every pair does the same MMA work whatever the tile
// count; a tile cut between pairs is finished by the last of them to
// arrive, which adds the fp32 partials in K order.
//
// Warp roles of ll_f8_kernel (7 warps): 0 TMA producer (both CTAs), 1 MMA
// issuer (leader) and TMEM allocator, 2-5 epilogue (lane quadrant
// warp % 4), 6 tile scheduler (leader) or slot-release forwarder (peer).
#pragma once
#include <cstdint>
#include <cuda.h>

#include "ll_kernels.cuh"
#include "ptx.cuh"

namespace llk {

// ============================================================ split of x
// Exponent e of the smallest power of two with a <= 448 * 2^e, from the
// bits of a non-negative bf16 value (448 = 1.75 * 2^8), limited to
// [-126, 126]; 0 for a == 0.
__device__ __forceinline__ int token_exp_from_bf16(uint32_t a16) {
  if (a16 == 0) return 0;
  const uint32_t bits = a16 << 16;
  const int E = static_cast<int>((bits >> 23) & 0xFFu);
  if (E == 0) return -126;  // below 2^-126: far below the clamp
  int e = E - 127 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return max(-126, min(126, e));
}

// Codes of eight bf16 values (one 16-byte chunk) scaled by `mult`.
__device__ __forceinline__ void xsplit_chunk(const uint4 v, float mult, int terms, uint2& hi, uint2& lo) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float u[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    u[2 * j] = __uint_as_float(w[j] << 16) * mult;  // exact: a power-of-two scaling
    u[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u) * mult;
  }
  uint16_t h[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = f32x2_to_e4m3x2(u[2 * j], u[2 * j + 1]);
  hi = make_uint2(h[0] | (static_cast<uint32_t>(h[1]) << 16), h[2] | (static_cast<uint32_t>(h[3]) << 16));
  if (terms == 2) {
    uint16_t l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 d = e4m3x2_to_f32x2(h[j]);
      // exact: u and its nearest e4m3 value differ by less than a quarter
      // of u's binade, on u's own grid
      l[j] = f32x2_to_e4m3x2(u[2 * j] - d.x, u[2 * j + 1] - d.y);
    }
    lo = make_uint2(l[0] | (static_cast<uint32_t>(l[1]) << 16), l[2] | (static_cast<uint32_t>(l[3]) << 16));
  }
}

__device__ __forceinline__ uint32_t absmax_bf16x8(uint32_t mx, const uint4 v) {
  mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
  mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
  mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
  return __vmaxu2(mx, v.w & 0x7FFF7FFFu);
}

// x [M, K] bf16 -> e_tok [M], xh [M, K] and (terms == 2) xl [M, K] e4m3fn.
// One warp per row.  Rows of up to 2048 values stay in registers between
// the maximum and the codes (one pass over global memory); longer rows are
// read twice, eight 16-byte loads in flight per lane.
constexpr int kXsRegChunks = 8;  // 16-byte chunks per lane held in registers
__global__ void __launch_bounds__(256) ll_xsplit_kernel(const uint16_t* __restrict__ x, int M, int K, int terms,
                                                        int* __restrict__ e_tok, uint8_t* __restrict__ xh,
                                                        uint8_t* __restrict__ xl) {
  // The down-projection launched after this kernel reads x only until its
  // epilogue: let it start now.
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nv = K >> 3;  // 16-byte chunks (8 bf16) per row
  const bool in_regs = nv <= 32 * kXsRegChunks;
  for (int m = blockIdx.x * wpb + (threadIdx.x >> 5); m < M; m += gridDim.x * wpb) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K);
    uint2* hr = reinterpret_cast<uint2*>(xh + static_cast<size_t>(m) * K);
    uint2* lr = terms == 2 ? reinterpret_cast<uint2*>(xl + static_cast<size_t>(m) * K) : nullptr;
    uint32_t mx = 0;  // |x| as bf16 bit patterns, two per word (order of the bits = order of the values)
    uint4 v[kXsRegChunks];
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kXsRegChunks; ++j)
        v[j] = lane + 32 * j < nv ? __ldg(xr + lane + 32 * j) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < kXsRegChunks; ++j) mx = absmax_bf16x8(mx, v[j]);
    } else {
      for (int i0 = lane; i0 < nv; i0 += 32 * kXsRegChunks) {
#pragma unroll
        for (int j = 0; j < kXsRegChunks; ++j)
          v[j] = i0 + 32 * j < nv ? __ldg(xr + i0 + 32 * j) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kXsRegChunks; ++j) mx = absmax_bf16x8(mx, v[j]);
      }
    }
    mx = max(mx & 0xFFFFu, mx >> 16);
    mx = __reduce_max_sync(0xffffffffu, mx);
    const int e = token_exp_from_bf16(mx);
    const float mult = exp2_int(-e);
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kXsRegChunks; ++j) {
        const int i = lane + 32 * j;
        if (i >= nv) break;
        uint2 h, l;
        xsplit_chunk(v[j], mult, terms, h, l);
        hr[i] = h;
        if (terms == 2) lr[i] = l;
      }
    } else {
      for (int i0 = lane; i0 < nv; i0 += 32 * kXsRegChunks) {
#pragma unroll
        for (int j = 0; j < kXsRegChunks; ++j)
          v[j] = i0 + 32 * j < nv ? __ldg(xr + i0 + 32 * j) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kXsRegChunks; ++j) {
          const int i = i0 + 32 * j;
          if (i >= nv) break;
          uint2 h, l;
          xsplit_chunk(v[j], mult, terms, h, l);
          hr[i] = h;
          if (terms == 2) lr[i] = l;
        }
      }
    }
    if (lane == 0) e_tok[m] = e;
  }
}

// ============================================== fused FP8-operand kernel
struct F8Params {
  CUtensorMap tm_xh;   // u8 hi [M, K]        box {128, 128}, 128B swizzle
  CUtensorMap tm_xl;   // u8 lo [M, K]        (terms == 2)
  CUtensorMap tm_q;    // u8 Q  [N, K]        box {128, 128}, 128B swizzle (rows of zero scale cleared)
  CUtensorMap tm_ahi;  // bf16 A'_hi [N, r_pad] box {32, 128}, 64B swizzle
  CUtensorMap tm_alo;  // bf16 A'_lo [N, r_pad]
  CUtensorMap tm_thi;  // bf16 t'_hi [M, r_pad] box {32, 128}, 64B swizzle
  CUtensorMap tm_tlo;  // bf16 t'_lo [M, r_pad]
  CUtensorMap tm_y;    // bf16 y [M, N]       box {32, 32}, 64B swizzle
  const int* e_tok;      // [M] token exponents
  const float* scale;    // [N] effective per-row scale
  const uint16_t* bias;  // [N] bf16 bits, or nullptr
  float* part;           // [2 * clusters][2] fp32 partial tiles of K-split tiles (layout: f8_part_at)
  int* cnt;              // [n_tiles][2][4] arrivals on a split tile (0 between launches)
  int* sched;            // [2]: tile counter, finished-leader counter (0 between launches)
  int M, N, K, r_pad;
  int terms;             // 1: hi only (FP8 activations); 2: hi + lo
  int n_ttiles, n_ftiles;  // 256-token and 256-feature tiles
  int clusters;          // CTA pairs of the grid
  int dp_waves;          // data-parallel waves of whole tiles before the stream-K tiles
  int lr_from_primary;   // 1: t' is written by the preceding kernel
  int withhold;          // debug: the producers issue nothing, so every consumer's wait runs out
  Watch watch;
};

constexpr int kF8Tile = 128 * 128;        // one CTA's 128 rows x 128 codes (16 KB)
constexpr int kF8LrBytes = 4 * 128 * 32 * 2;  // t'_hi, t'_lo, A'_hi, A'_lo chunks of 32 (32 KB)
constexpr int kF8Ring = 192 * 1024;
constexpr int kF8MaxStages = 6;
constexpr int kF8EpiWarps = 4;
constexpr int kF8SchedWarp = 2 + kF8EpiWarps;
constexpr int kF8Threads = 32 * (kF8SchedWarp + 1);
constexpr int kF8TileRing = 2;
// The leader's producer asks for the next tile this many K steps before
// the end of its current one, so a pair claims a tile only when it is about
// to load it: pairs that start late (their SMs still held by the kernels
// before) or run slow take fewer tiles instead of finding them claimed.
constexpr int kF8ReqAhead = 3;
constexpr int kF8EpiWarp = 2 * 32 * 64 + 256 * 8;  // per epilogue warp: two 32 x 32 bf16 staging buffers,
                                                     // then the tile's 256 (scale, bias) pairs
constexpr int kF8Epi = kF8EpiWarps * kF8EpiWarp;
constexpr int kF8Group = 8;                        // token tiles per raster group
constexpr int kF8PartFloats = 128 * 256;           // one CTA's partial tile

// float4 index of (row, columns 32 * chunk + 4 * k .. + 3) in a CTA's
// partial tile: the 32 rows of a warp's quadrant are adjacent for each
// (chunk, k), so each of the warp's float4 stores and loads is one
// contiguous 512-byte run.
__device__ __forceinline__ int f8_part_at(int row, int chunk, int k) { return (chunk * 8 + k) * 128 + row; }

__host__ __device__ constexpr int f8_stage_bytes(int terms) { return (terms + 1) * kF8Tile; }
__host__ __device__ constexpr int f8_stages(int terms) {
  return kF8Ring / f8_stage_bytes(terms) < kF8MaxStages ? kF8Ring / f8_stage_bytes(terms) : kF8MaxStages;
}
__host__ __device__ constexpr int f8_smem_bytes() { return kF8Ring + kF8Epi + 1024 + 256; }

__device__ __forceinline__ void f8_tile_coords(const F8Params& p, int T, int& tt, int& ft) {
  const int per_group = kF8Group * p.n_ftiles;
  const int g = T / per_group;
  const int first = g * kF8Group;
  const int gsize = min(kF8Group, p.n_ttiles - first);
  const int idx = T - g * per_group;
  ft = idx / gsize;
  tt = first + idx % gsize;
}

// Work split.  With C CTA pairs and n tiles, the first D waves (chosen on
// the host, normally n / C - (0 or 1)) are data-parallel: the pairs take whole tiles from a device-wide
// counter in a grouped raster order, so the tiles in flight are neighbours
// that share their x and Q slabs in L2 and a pair that starts late takes
// fewer.  The remaining S = n - D * C tiles (one partial wave, merged with
// the last full wave when it is short) are split stream-K: their
// (tile, 128-wide K step) units, tile-major, are cut into C equal
// contiguous ranges, one per pair, so every pair ends at the same time.  A
// range is cut further at tile boundaries into segments (T, k0, k1).  A
// tile whose K steps fall into several ranges ("split tile") is finished
// by the last of its pairs to arrive.
struct F8Split {
  int C, nS, DT, S, U;  // pairs, K steps, data-parallel tiles, stream-K tiles, stream-K units
  __device__ F8Split(int n_tiles, int C_, int nS_, int D) : C(C_), nS(nS_) {
    DT = min(n_tiles, D * C);
    S = n_tiles - DT;
    U = S * nS;
  }
  __device__ int begin(int c) const { return static_cast<int>(static_cast<long long>(U) * c / C); }
  // Pair that holds stream-K unit u.
  __device__ int owner(int u) const {
    int c = static_cast<int>(static_cast<long long>(u) * C / U);
    while (c + 1 < C && begin(c + 1) <= u) ++c;
    while (c > 0 && begin(c) > u) --c;
    return c;
  }
  // Partial slot of pair j's segment on stream-K tile Ts: 2j for its first
  // segment, 2j + 1 for its last when that is another one.
  __device__ int slot(int j, int Ts) const { return 2 * j + (begin(j) < Ts * nS ? 1 : 0); }
};
struct F8Seg {
  int T, k0, k1;
  bool dyn;  // a whole tile taken from the scheduler's ring
};
// This CTA's view of the tile ring filled by the leader's scheduler.
struct F8TileRing {
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
    if (++ti == kF8TileRing) { ti = 0; tph ^= 1; }
    return T >= 0;
  }
};

// This pair's segments in order: whole tiles from the ring while the
// data-parallel waves last, then its stream-K range.
struct F8Sched {
  const F8Split& sp;
  F8TileRing tr;
  bool dp_done = false;
  int c, u, u_end;
  __device__ F8Sched(const F8Split& sp_, int c_) : sp(sp_), c(c_), u(sp_.begin(c_)), u_end(sp_.begin(c_ + 1)) {}
  int wv = 0;  // whole tiles taken so far (static first waves)
  __device__ bool next(F8Seg& g, uint64_t* tile_full, uint64_t* tile_empty, int* tile_slot, const Watch& w,
                       int code, bool whole_warp) {
    if (!dp_done && sp.S > 0) {
      // With a stream-K tail the whole tiles are dealt out statically
      // (pair c: c, C + c, ...), so every pair reaches its stream-K range
      // after the same amount of work.
      if (wv * sp.C + c < sp.DT) {
        g.T = wv * sp.C + c;
        g.k0 = 0;
        g.k1 = sp.nS;
        g.dyn = false;
        ++wv;
        return true;
      }
      dp_done = true;
    }
    if (!dp_done) {
      int T;
      if (tr.next(tile_full, tile_empty, tile_slot, w, code, whole_warp, T)) {
        g.T = T;
        g.k0 = 0;
        g.k1 = sp.nS;
        g.dyn = true;
        return true;
      }
      dp_done = true;
    }
    if (u >= u_end) return false;
    const int Ts = u / sp.nS;
    g.T = sp.DT + Ts;
    g.k0 = u - Ts * sp.nS;
    g.k1 = min(sp.nS, g.k0 + (u_end - u));
    g.dyn = false;
    u += g.k1 - g.k0;
    return true;
  }
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// kAct: kActNone, kActGelu, or kActGeglu (y = h * gelu(g) over the halves of
// each tile's features; tm_y is then [M, N/2]).
template <int kAct>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kF8Threads, 1)
    ll_f8_kernel(const __grid_constant__ F8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* ring = smem;
  uint8_t* epi = ring + kF8Ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kF8Epi);  // leader: both CTAs' loads landed
  uint64_t* empty = full + kF8MaxStages;                      // both: the MMAs are done with the slot
  uint64_t* tfull = empty + kF8MaxStages;                     // both: accumulator buffer ready
  uint64_t* tempty = tfull + 2;                               // leader: both CTAs' epilogues done
  uint64_t* tile_full = tempty + 2;
  uint64_t* tile_empty = tile_full + kF8TileRing;
  uint64_t* drain = tile_empty + kF8TileRing;
  uint64_t* tile_req = drain + 1;  // leader: its producer wants the next tile
  int* tile_slot = reinterpret_cast<int*>(tile_req + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_slot + kF8TileRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int terms = p.terms;
  const int sb = f8_stage_bytes(terms);
  const int ns = f8_stages(terms);
  const int nS = (p.K + 127) / 128;  // K steps of 128 (a step past K loads as zeros)
  const int nR = p.r_pad / 32;       // low-rank chunks of 32
  const int cid = static_cast<int>(blockIdx.x >> 1);
  const F8Split sp(p.n_ttiles * p.n_ftiles, p.clusters, nS, p.dp_waves);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF8MaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kF8EpiWarps);
    }
    for (int s = 0; s < kF8TileRing; ++s) {
      mbar_init(&tile_full[s], 1);
      // readers: producer + epilogue warps (+ MMA issuer and the peer's forwarder on the leader)
      mbar_init(&tile_empty[s], 1 + kF8EpiWarps + (leader ? 2 : 0));
    }
    mbar_init(drain, 1);
    mbar_init(tile_req, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_xh);
    if (terms == 2) tma_prefetch_desc(&p.tm_xl);
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
    // ------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
      int slot = 0;
      uint32_t ph = 0;
      bool ok = true, issued = false, waited = false;
      F8Sched sch(sp, cid);
      F8Seg g;
      while (ok && sch.next(g, tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutProducer, false)) {
        if (p.withhold) { ok = false; break; }  // debug: no loads, the consumers time out
        int tt, ft;
        f8_tile_coords(p, g.T, tt, ft);
        const int t0 = tt * 256 + 128 * static_cast<int>(rank);
        const int f0 = ft * 256 + 128 * static_cast<int>(rank);
        for (int s = g.k0; s < g.k1; ++s) {
          if (!mbar_wait(&empty[slot], ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[slot], 2u * sb);
          uint8_t* dst = ring + slot * sb;
          const uint32_t bar = full0 + 8u * slot;
          tma_load_2d_pair(dst, &p.tm_xh, bar, s * 128, t0);
          if (terms == 2) tma_load_2d_pair(dst + kF8Tile, &p.tm_xl, bar, s * 128, t0);
          tma_load_2d_pair(dst + terms * kF8Tile, &p.tm_q, bar, s * 128, f0);
          issued = true;
          if (leader && g.dyn && s == max(g.k0, g.k1 - kF8ReqAhead)) mbar_arrive(tile_req);
          if (++slot == ns) { slot = 0; ph ^= 1; }
        }
        if (g.k0 != 0) continue;  // the low-rank term goes with a tile's first K steps
        if (ok && nR > 0 && !waited && p.lr_from_primary) {
          pdl_wait_primary();
          waited = true;
        }
        for (int jb = 0; jb < nR && ok; ++jb) {
          if (!mbar_wait(&empty[slot], ph ^ 1, p.watch, kErrTimeoutProducer)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[slot], 2u * kF8LrBytes);
          uint8_t* dst = ring + slot * sb;
          const uint32_t bar = full0 + 8u * slot;
          tma_load_2d_pair(dst, &p.tm_thi, bar, jb * 32, t0);
          tma_load_2d_pair(dst + 8192, &p.tm_tlo, bar, jb * 32, t0);
          tma_load_2d_pair(dst + 16384, &p.tm_ahi, bar, jb * 32, f0);
          tma_load_2d_pair(dst + 24576, &p.tm_alo, bar, jb * 32, f0);
          issued = true;
          if (++slot == ns) { slot = 0; ph ^= 1; }
        }
      }
      if (!ok && issued) {
        // Loads already issued must land before the CTA exits; they
        // complete on leader barriers whose other arrivals may never come
        // now, so wait a bounded settle time far above any load latency.
        const uint64_t c0 = clock_cycles();
        while (clock_cycles() - c0 < 400000ull) {  // >= 200 us at any clock up to 2 GHz
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // --------------------------------------------- MMA issuer (leader)
      const uint32_t id8 = idesc_e4m3(256, 256);
      const uint32_t id16 = idesc_bf16(256, 256);
      int slot = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      F8Sched sch(sp, cid);
      F8Seg g;
      while (ok && sch.next(g, tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutMma, false)) {
        const int buf = it & 1;
        if (!mbar_wait_cl(&tempty[buf], ((it >> 1) & 1) ^ 1, p.watch, kErrTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d = tbase + 256u * buf;
        for (int s = g.k0; s < g.k1; ++s) {
          if (!mbar_wait_cl(&full[slot], ph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(ring + slot * sb);
          const uint64_t dh = sdesc_kmajor_sw128(base);
          const uint64_t dl = sdesc_kmajor_sw128(base + kF8Tile);
          const uint64_t dq = sdesc_kmajor_sw128(base + terms * kF8Tile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_f8_pair(d, dh + 2 * kk, dq + 2 * kk, id8, (s != g.k0 || kk != 0) ? 1u : 0u);
            if (terms == 2) mma_f8_pair(d, dl + 2 * kk, dq + 2 * kk, id8, 1u);
          }
          tc_commit_pair(&empty[slot], 0x3);
          if (++slot == ns) { slot = 0; ph ^= 1; }
        }
        for (int jb = 0; g.k0 == 0 && jb < nR && ok; ++jb) {
          if (!mbar_wait_cl(&full[slot], ph, p.watch, kErrTimeoutMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(ring + slot * sb);
          const uint64_t th = sdesc_kmajor_sw64(base), tl = sdesc_kmajor_sw64(base + 8192);
          const uint64_t ah = sdesc_kmajor_sw64(base + 16384), al = sdesc_kmajor_sw64(base + 24576);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            mma_ss_pair(d, th + 2 * kk, ah + 2 * kk, id16, 1u);  // t'_hi A'_hi
            mma_ss_pair(d, tl + 2 * kk, ah + 2 * kk, id16, 1u);  // t'_lo A'_hi
            mma_ss_pair(d, th + 2 * kk, al + 2 * kk, id16, 1u);  // t'_hi A'_lo
          }
          tc_commit_pair(&empty[slot], 0x3);
          if (++slot == ns) { slot = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(&tfull[buf], 0x3);
        ++it;
      }
      // No MMA may still run when TMEM is released.
      tc_commit_pair(drain, 0x1);
      mbar_wait_drain(drain, 0, p.watch);
    }
  } else if (warp < kF8SchedWarp) {
    // ------------------------------------------------------------ epilogue
    // TMEM lane = token row of this CTA; column = feature of the tile.
    const int q = warp & 3;
    const int row = 32 * q + lane;
    uint8_t* stg = epi + (warp - 2) * kF8EpiWarp;
    float2* prm = reinterpret_cast<float2*>(stg + 2 * 32 * 64);
    const uint32_t tl = tbase + ((32u * q) << 16);
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    const int sw = (lane >> 1) & 3;  // 64-byte swizzle phase of this lane's staging row
    int it = 0, eb = 0;
    F8Sched sch(sp, cid);
    F8Seg g;
    while (sch.next(g, tile_full, tile_empty, tile_slot, p.watch, kErrTimeoutEpilogue, true)) {
      int tt, ft;
      f8_tile_coords(p, g.T, tt, ft);
      const int buf = it & 1;
      const int trow = tt * 256 + 128 * static_cast<int>(rank) + 32 * q;
      const int tok = trow + lane;
      const int fbase = ft * 256;
      const bool split = g.k0 != 0 || g.k1 != nS;
      // The tile's per-feature (scale, bias) into this warp's shared
      // buffer and this row's token scale, loaded before the wait so that
      // their latency hides under the MMAs.
      {
        float sl[8], bl[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int fl = fbase + 32 * c + lane;
          sl[c] = fl < p.N ? __ldg(p.scale + fl) : 0.f;
          bl[c] = (p.bias != nullptr && fl < p.N) ? bf16_bits_to_float(__ldg(p.bias + fl)) : 0.f;
        }
        __syncwarp();  // the previous tile's chunks are done with the buffer
#pragma unroll
        for (int c = 0; c < 8; ++c) prm[32 * c + lane] = make_float2(sl[c], bl[c]);
        __syncwarp();
      }
      const float sm = tok < p.M ? exp2_int(__ldg(p.e_tok + tok)) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (it >> 1) & 1, p.watch, kErrTimeoutEpilogue))) break;
      tc_fence_after();
      const uint32_t acc = tl + 256u * buf;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(&tempty[buf]);
          else
            mbar_arrive_cluster(tempty_leader + 8u * buf);
        }
      };
      // Pairs holding a split tile: first and last (inclusive), and this
      // pair's position among them.
      int c_first = 0, c_last = 0;
      const int Ts = g.T - sp.DT;  // index among the stream-K tiles
      if (split) {
        c_first = sp.owner(Ts * nS);
        c_last = sp.owner(Ts * nS + nS - 1);
        // This pair's fp32 partial of its own rows, in case another pair
        // arrives last.
        float4* dst = reinterpret_cast<float4*>(
            p.part + (static_cast<size_t>(sp.slot(cid, Ts)) * 2 + rank) * kF8PartFloats);
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld32_wait(acc + 32u * c, v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            __stcg(dst + f8_part_at(row, c, i),
                   make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                               __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
        }
        __threadfence();
        __syncwarp();
        int old = 0;
        int* cnt = p.cnt + (g.T * 2 + static_cast<int>(rank)) * 4 + q;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != c_last - c_first) {  // another pair finishes this tile
          release();
          ++it;
          continue;
        }
        __threadfence();  // acquire: the other pairs' partials are visible
        if (lane == 0) *cnt = 0;
      }
      if constexpr (kAct == kActGeglu) {
        // GEGLU: the set-time order puts the gate rows of output features
        // fbase/2 + j (j < 128) at tile columns 128 + j, beside their value
        // rows at columns j, so each thread has both for its token.  Whole
        // tiles only (the host keeps the stream-K tail off).
        for (int c = 0; c < 4; ++c) {
          uint32_t vh[32], vg[32];
          tmem_ld32x2_wait(acc + 32u * c, vh, acc + 128u + 32u * c, vg);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 h0 = prm[32 * c + 2 * i], h1 = prm[32 * c + 2 * i + 1];
            const float2 g0 = prm[128 + 32 * c + 2 * i], g1 = prm[128 + 32 * c + 2 * i + 1];
            const float o0 = fmaf(h0.x * sm, __uint_as_float(vh[2 * i]), h0.y) *
                             gelu_tanh(fmaf(g0.x * sm, __uint_as_float(vg[2 * i]), g0.y));
            const float o1 = fmaf(h1.x * sm, __uint_as_float(vh[2 * i + 1]), h1.y) *
                             gelu_tanh(fmaf(g1.x * sm, __uint_as_float(vg[2 * i + 1]), g1.y));
            w[i] = pack_bf16x2(o0, o1);
          }
          if (lane == 0) tma_store_wait_read<1>();
          __syncwarp();
          uint8_t* st = stg + eb * (32 * 64);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(st + lane * 64 + 16 * (j ^ sw)) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int fo = fbase / 2 + 32 * c;
            if (trow < p.M && fo < p.N / 2) tma_store_2d(&p.tm_y, st, fo, trow);
            tma_store_commit();
          }
          eb ^= 1;
        }
        release();
        ++it;
      } else {
        // A split tile's other pairs' partials, four chunks (128 columns) of
        // one pair per batch of loads, so a finish costs a few L2 round trips
        // instead of one per chunk.
        float4 pf[4][8];
        for (int c0 = 0; c0 < 8; c0 += 4)
  #pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = c0 + cc;
          // Sum of the pairs' terms in K order, starting from zero (a fixed
          // order, whichever pair arrives last); this pair's own term comes
          // from TMEM.
          uint32_t v[32];
          tmem_ld32_wait(acc + 32u * c, v);
          float a[32];
  #pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = split ? 0.f : __uint_as_float(v[i]);
          for (int j = c_first; split && j <= c_last; ++j) {
            if (j == cid) {
  #pragma unroll
              for (int i = 0; i < 32; ++i) a[i] += __uint_as_float(v[i]);
              continue;
            }
            if (c_last - c_first == 1 && cc == 0) {
              // two pairs: prefetch the other's next four chunks at once
              const float4* s4 = reinterpret_cast<const float4*>(
                  p.part + (static_cast<size_t>(sp.slot(j, Ts)) * 2 + rank) * kF8PartFloats);
  #pragma unroll
              for (int c2 = 0; c2 < 4; ++c2)
  #pragma unroll
                for (int i = 0; i < 8; ++i) pf[c2][i] = __ldcg(s4 + f8_part_at(row, c0 + c2, i));
            }
            float4 u[8];
            if (c_last - c_first == 1) {
  #pragma unroll
              for (int i = 0; i < 8; ++i) u[i] = pf[cc][i];
            } else {
              const float4* s4 = reinterpret_cast<const float4*>(
                  p.part + (static_cast<size_t>(sp.slot(j, Ts)) * 2 + rank) * kF8PartFloats);
  #pragma unroll
              for (int i = 0; i < 8; ++i) u[i] = __ldcg(s4 + f8_part_at(row, c, i));
            }
  #pragma unroll
            for (int i = 0; i < 8; ++i) {
              a[4 * i] += u[i].x; a[4 * i + 1] += u[i].y; a[4 * i + 2] += u[i].z; a[4 * i + 3] += u[i].w;
            }
          }
          uint32_t w[16];
  #pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 p0 = prm[32 * c + 2 * i], p1 = prm[32 * c + 2 * i + 1];  // broadcast reads
            w[i] = pack_bf16x2(epi_act<kAct>(fmaf(p0.x * sm, a[2 * i], p0.y)),
                               epi_act<kAct>(fmaf(p1.x * sm, a[2 * i + 1], p1.y)));
          }
          if (lane == 0) tma_store_wait_read<1>();
          __syncwarp();
          uint8_t* st = stg + eb * (32 * 64);
  #pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(st + lane * 64 + 16 * (j ^ sw)) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (trow < p.M && fbase + 32 * c < p.N) tma_store_2d(&p.tm_y, st, fbase + 32 * c, trow);
            tma_store_commit();
          }
          eb ^= 1;
        }
        release();
        ++it;
      }
    }
    if (lane == 0) tma_store_wait<0>();
  } else if (lane == 0) {
    const int dp_tiles = sp.DT;
    if (leader) {
      // ----------------------------------- tile scheduler (leader): the
      // data-parallel tiles.  A slot is refilled once this CTA's readers and
      // the peer's forwarder have released it; the tile number goes into
      // both CTAs' slots, the peer's by a cluster store ordered before the
      // release arrival on the peer's barrier.
      const uint32_t peer_slot = mapa_shared(smem_u32(&tile_slot[0]), 1);
      const uint32_t peer_full = mapa_shared(smem_u32(&tile_full[0]), 1);
      int ti = 0;
      uint32_t tph = 0, rph = 0;
      for (bool first = true;; first = false) {
        if (!mbar_wait_cl(&tile_empty[ti], tph ^ 1, p.watch, kErrTimeoutProducer)) break;
        // every claim after the first waits for the producer's request
        if (!first) {
          if (!mbar_wait(tile_req, rph, p.watch, kErrTimeoutProducer)) break;
          rph ^= 1;
        }
        // (no dynamic tiles when a stream-K tail deals them out statically)
        const int got = dp_tiles > 0 && sp.S == 0 ? atomicAdd(&p.sched[0], 1) : dp_tiles;
        const int T = got < dp_tiles ? got : -1;
        *reinterpret_cast<volatile int*>(&tile_slot[ti]) = T;
        st_shared_cluster_u32(peer_slot + 4u * ti, static_cast<uint32_t>(T));
        mbar_arrive_cluster_release(peer_full + 8u * ti);
        mbar_arrive(&tile_full[ti]);
        if (++ti == kF8TileRing) { ti = 0; tph ^= 1; }
        if (T < 0) break;
      }
      // The last leader to finish resets the scheduler for the next launch.
      __threadfence();
      if (atomicAdd(&p.sched[1], 1) == static_cast<int>(gridDim.x / 2) - 1) {
        atomicExch(&p.sched[0], 0);
        atomicExch(&p.sched[1], 0);
      }
    } else {
      // -------------------------------- slot-release forwarder (peer)
      const uint32_t leader_empty = mapa_shared(smem_u32(&tile_empty[0]), 0);
      int ti = 0;
      uint32_t tph = 0;
      for (;;) {
        if (!mbar_wait_cl(&tile_full[ti], tph, p.watch, kErrTimeoutProducer)) break;
        const int T = *reinterpret_cast<volatile int*>(&tile_slot[ti]);
        if (T < 0) break;  // the last slot: nothing refills it
        if (!mbar_wait_cl(&tile_empty[ti], tph, p.watch, kErrTimeoutProducer)) break;
        mbar_arrive_cluster_release(leader_empty + 8u * ti);
        if (++ti == kF8TileRing) { ti = 0; tph ^= 1; }
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
