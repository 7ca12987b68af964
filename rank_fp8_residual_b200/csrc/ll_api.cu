// Host side of the C ABI declared in include/rank_fp8_residual.h:
// argument validation, handle-owned device copies of the factors, TMA
// tensor-map construction, workspace management and the kernel chain of
// one forward (kernels in ll_kernels.cuh and ll_tc.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/rank_fp8_residual.h"
#include "ll_kernels.cuh"
#include "ll_tc.cuh"
#include "ll_tc2.cuh"
#include "ll_stream.cuh"
#include "ll_f8.cuh"
#include "ll_f8_stream.cuh"
#include "ll_gemv.cuh"
#include "ll_decompose.cuh"

namespace {

thread_local int g_last_error = LL_OK;

int fail(int code) {
  g_last_error = code;
  return code;
}

// ------------------------------------------------ driver entry point (TMA)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols], row pitch `pitch_bytes`; box =
// {box_cols, box_rows}.  Elements outside the tensor load as zeros.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
              uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

// 3-D view {d0, d1, d2} with strides {s1, s2} (bytes) and box {b0, b1, b2}:
// used to read several 64-wide K chunks of a row-major matrix in one load
// (d0 = 64 elements of a chunk, d1 = rows, d2 = chunk index).
bool make_map3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device memory (or managed memory) of device `dev`.
bool is_device_ptr_on(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

// Stored row of original output feature n.  With a GEGLU epilogue, tile t
// of 256 stored rows holds the value features 128t .. 128t + 127 and then
// their gate features N/2 + 128t .. (so both halves of an output feature
// meet in one thread of the FP8-operand kernel's epilogue); otherwise the
// identity.
int original_row(int stored, int N, bool geglu) {
  if (!geglu) return stored;
  const int t = stored / 256, i = stored % 256;
  return i < 128 ? 128 * t + i : N / 2 + 128 * t + (i - 128);
}

// Device-to-device copy of N rows of `width` bytes into the stored order.
bool copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, int N, bool geglu) {
  if (!geglu)
    return cudaMemcpy2D(dst, dpitch, src, spitch, width, N, cudaMemcpyDeviceToDevice) == cudaSuccess;
  bool ok = true;
  for (int t = 0; t < N / 256; ++t)
    for (int half = 0; half < 2; ++half) {
      const int src_row = half == 0 ? 128 * t : N / 2 + 128 * t;
      ok &= cudaMemcpy2D(static_cast<char*>(dst) + (256 * t + 128 * half) * dpitch, dpitch,
                         static_cast<const char*>(src) + src_row * spitch, spitch, width, 128,
                         cudaMemcpyDeviceToDevice) == cudaSuccess;
    }
  return ok;
}

// Byte ranges [a, a + na) and [b, b + nb) intersect.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const char* pa = static_cast<const char*>(a);
  const char* pb = static_cast<const char*>(b);
  return na > 0 && nb > 0 && pa < pb + nb && pb < pa + na;
}

int next_pow2_ge32(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

}  // namespace

// Joint plan of the single-CTA fused kernel and the down-projection.
struct TcChoice {
  int bt;  // tokens per fused-kernel tile
  int ks;  // K splits of the down-projection (1 when r == 0)
};

// TMA descriptors that depend on the call's x, y and M (and on the
// workspace, whose growth clears them).
struct CallMaps {
  const void* c_x = nullptr;
  void* c_yptr = nullptr;
  int c_M = -1;
  bool c_f8 = false;  // the FP8-operand maps are built
  CUtensorMap c_x128, c_x256, c_y, c_thi128, c_tlo128, c_thi256, c_tlo256;
  CUtensorMap c_xs, c_this, c_tlos;     // streaming kernel: x and t boxes of Mt rows
  CUtensorMap c_xbt, c_thibt, c_tlobt;  // fused single-CTA kernel: x and t boxes of bt rows
  int c_bt = 0;
  CUtensorMap c_x2p, c_thip, c_tlop;  // CTA-pair kernel: x and t boxes of bt2 / 2 rows
  int c_bt2 = 0;
  CUtensorMap c_xh, c_xl, c_thi32, c_tlo32, c_y64;  // FP8-operand kernel
  CUtensorMap c_xhs, c_xls;                         // FP8-operand streaming kernel: code boxes of Mt rows
};
constexpr int kMapCache = 8;  // descriptor sets kept per layer (e.g. the chunks of a host-buffer forward)

struct ll_layer {
  int N = 0, K = 0, r = 0, r_pad = 0, klr = 64, scale_mode = 0;
  int device = 0, num_sms = 0;
  bool ready = false;
  bool has_bias = false;
  // factors (device, handle-owned)
  uint8_t* Q = nullptr;       // [N, K] e4m3fn codes as given
  uint8_t* Qf = nullptr;      // rows with zero scale cleared (== Q when no scale is zero)
  uint16_t* A = nullptr;      // [N, r_pad] bf16, zero-padded
  uint16_t* Ahi = nullptr;    // [N, r_pad] bf16 of A / s_eff
  uint16_t* Alo = nullptr;    // [N, r_pad] bf16 of A / s_eff - Ahi
  uint16_t* B = nullptr;      // [r_pad, K] bf16, zero-padded
  float* scale = nullptr;     // [N] scale as given (broadcast for per-tensor)
  float* scale_eff = nullptr; // [N] scale, 1 where the scale is zero
  uint16_t* bias = nullptr;   // [N]
  int* status = nullptr;      // device status word
  int* flags = nullptr;       // [2] set-time scan flags
  int* sched = nullptr;       // [2] tile scheduler of the fused kernel
  // workspace for t
  int ws_M = 0;
  uint16_t* t_hi = nullptr;
  uint16_t* t_lo = nullptr;
  // FP8-operand path: per-token exponents and e4m3 codes of x
  int ws8_M = 0;
  int* e_tok = nullptr;
  uint8_t* xh = nullptr;
  uint8_t* xl = nullptr;
  int* f8_cnt = nullptr;     // arrival counters of K-split tiles, [tiles of ws8_M rows][2][4]
  size_t f8_cnt_n = 0;
  float* f8_part = nullptr;  // fp32 partial tiles, two slots per CTA pair
  float* t32 = nullptr;      // GEMV path: t in fp32, [kGvMaxM, r_pad]
  CUtensorMap tm_q128, tm_ahi32, tm_alo32;     // set-time maps of the FP8-operand kernel
  mutable int f8_clusters = 0;                 // co-resident clusters of the FP8-operand kernel
  // host-buffer forward staging: device copies of x and y, and two copy
  // streams (host to device, device to host) that overlap the chunks' copies
  // with the forwards on the caller's stream
  void* dx = nullptr;
  void* dy = nullptr;
  size_t dx_bytes = 0, dy_bytes = 0;
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t hev[2 * 8 + 2] = {};  // start, copy-in done [8], forward done [8], copy-out done
  // weight tensor maps
  CUtensorMap tm_q, tm_qf, tm_a, tm_ahi, tm_alo, tm_b;
  int b_box = 0;
  // per-call descriptors: the current set, and the last kMapCache sets built
  CallMaps cm;
  CallMaps cm_cache[kMapCache];
  int cm_next = 0;
  CUtensorMap tm_q3;  // 3-D view of the (row-cleared) residual, 4 K chunks per box
  CUtensorMap tm_q3b2;  // the same view, 2 K chunks per box (fused single-CTA kernel)
  mutable int tcp_M = -1;  // M of the cached joint plan (single-CTA kernel)
  mutable TcChoice tcp{};
  mutable int tcp2_M = -1;  // M of the cached joint plan (CTA-pair kernel)
  mutable TcChoice tcp2{};
  mutable int pair_clusters = 0;  // co-resident clusters of the CTA-pair kernel
  int variant = LL_VARIANT_AUTO;
  int epilogue = LL_EPILOGUE_NONE;  // activation fused into the epilogue
  int withhold = 0;
  uint64_t timeout_ns = 2000000000ull;
  int last_launches = 0;
  // profiling
  int profiling = 0;
  int prof_valid = 0;
  cudaEvent_t ev[8] = {};
  const char* names[8] = {};
};

namespace {

void free_layer_mem(ll_layer* h) {
  for (cudaEvent_t& e : h->ev)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t& e : h->hev)
    if (e) cudaEventDestroy(e);
  if (h->cin) cudaStreamDestroy(h->cin);
  if (h->cout) cudaStreamDestroy(h->cout);
  if (h->Qf && h->Qf != h->Q) cudaFree(h->Qf);
  cudaFree(h->Q);
  cudaFree(h->A);
  cudaFree(h->Ahi);
  cudaFree(h->Alo);
  cudaFree(h->B);
  cudaFree(h->scale);
  cudaFree(h->scale_eff);
  cudaFree(h->bias);
  cudaFree(h->status);
  cudaFree(h->flags);
  cudaFree(h->sched);
  cudaFree(h->t_hi);
  cudaFree(h->t_lo);
  cudaFree(h->dx);
  cudaFree(h->dy);
  cudaFree(h->e_tok);
  cudaFree(h->xh);
  cudaFree(h->xl);
  cudaFree(h->f8_cnt);
  cudaFree(h->f8_part);
  cudaFree(h->t32);
}

// The epilogue activation is a template parameter of each kernel (see
// epi_act): one instantiation per activation code.
using MainFn = void (*)(llk::MainParams);
using TcFn = void (*)(llk::TcParams);
using Tc2Fn = void (*)(llk::Tc2Params);
using StreamFn = void (*)(llk::StreamParams);
using F8Fn = void (*)(llk::F8Params);
MainFn kernel_main(int act) { return act == llk::kActGelu ? llk::ll_main_kernel<llk::kActGelu> : llk::ll_main_kernel<llk::kActNone>; }
TcFn kernel_tc(int act) { return act == llk::kActGelu ? llk::ll_tc_kernel<llk::kActGelu> : llk::ll_tc_kernel<llk::kActNone>; }
Tc2Fn kernel_tc2(int act) { return act == llk::kActGelu ? llk::ll_tc2_kernel<llk::kActGelu> : llk::ll_tc2_kernel<llk::kActNone>; }
StreamFn kernel_stream(int act) {
  return act == llk::kActGelu ? llk::ll_stream_kernel<llk::kActGelu> : llk::ll_stream_kernel<llk::kActNone>;
}
using F8sFn = void (*)(llk::F8sParams);
F8sFn kernel_f8s(int act) {
  return act == llk::kActGelu ? llk::ll_f8_stream_kernel<llk::kActGelu> : llk::ll_f8_stream_kernel<llk::kActNone>;
}
F8Fn kernel_f8(int act) {
  return act == llk::kActGeglu  ? llk::ll_f8_kernel<llk::kActGeglu>
         : act == llk::kActGelu ? llk::ll_f8_kernel<llk::kActGelu>
                                : llk::ll_f8_kernel<llk::kActNone>;
}

using GemvTFn = void (*)(const uint16_t*, const uint16_t*, float*, int, int);
using GemvFn = void (*)(llk::GemvParams);
template <int kM>
GemvFn gemv_kernel_m(int act) {
  return act == llk::kActGelu ? llk::ll_gemv_kernel<kM, llk::kActGelu> : llk::ll_gemv_kernel<kM, llk::kActNone>;
}
GemvFn kernel_gemv(int M, int act) {
  switch (M) {
    case 1: return gemv_kernel_m<1>(act);
    case 2: return gemv_kernel_m<2>(act);
    case 3: return gemv_kernel_m<3>(act);
    default: return gemv_kernel_m<4>(act);
  }
}
GemvTFn kernel_gemv_t(int M) {
  switch (M) {
    case 1: return llk::ll_gemv_t_kernel<1>;
    case 2: return llk::ll_gemv_t_kernel<2>;
    case 3: return llk::ll_gemv_t_kernel<3>;
    default: return llk::ll_gemv_t_kernel<4>;
  }
}

int set_smem_attrs_once() {
  static int rc = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    rc = 0;
    auto smem = [](auto f, size_t bytes) {
      if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
          cudaSuccess)
        rc = 1;
    };
    for (int a = 0; a < 2; ++a) {
      smem(kernel_main(a), llk::main_smem_bytes());
      smem(kernel_tc(a), llk::tc_smem_bytes());
      smem(kernel_tc2(a), llk::tc2_smem_bytes());
      smem(kernel_stream(a), llk::st_smem_max());
      smem(kernel_f8s(a), llk::ss_smem_max());
    }
    for (int a = 0; a < 3; ++a) smem(kernel_f8(a), llk::f8_smem_bytes());
    // The GEMV pair shares SMs while the t kernel runs: both ask for the
    // largest shared-memory carve-out, so an SM need not be reconfigured.
    auto carve = [](auto f) {
      if (cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) rc = 1;
    };
    for (int m = 1; m <= llk::kGvMaxM; ++m) {
      smem(kernel_gemv_t(m), 227 * 1024 - llk::kGvRingBytes);
      carve(kernel_gemv_t(m));
      for (int a = 0; a < 2; ++a) {
        smem(kernel_gemv(m, a), 227 * 1024);
        carve(kernel_gemv(m, a));
      }
    }
    smem(llk::ll_lrdown_kernel, llk::lr_smem_bytes(256));
  });
  return rc;
}

// Invalidates every descriptor set (the workspace they point into moved).
void clear_call_maps(ll_layer* h) {
  h->cm.c_M = -1;
  for (CallMaps& c : h->cm_cache) c.c_M = -1;
}

// Grow the t workspace to hold `M` rows (stream-ordered).
int ensure_workspace(ll_layer* h, int M, cudaStream_t st) {
  if (h->r_pad == 0) return LL_OK;
  if (M > h->ws_M) {
    int newM = std::max(M, h->ws_M * 3 / 2);
    newM = (newM + 255) / 256 * 256;
    uint16_t *th = nullptr, *tl = nullptr;
    const size_t bytes = static_cast<size_t>(newM) * h->r_pad * sizeof(uint16_t);
    if (cudaMallocAsync(reinterpret_cast<void**>(&th), bytes, st) != cudaSuccess ||
        cudaMallocAsync(reinterpret_cast<void**>(&tl), bytes, st) != cudaSuccess) {
      cudaGetLastError();
      if (th) cudaFreeAsync(th, st);
      return LL_ERR_OOM;
    }
    if (h->t_hi) cudaFreeAsync(h->t_hi, st);
    if (h->t_lo) cudaFreeAsync(h->t_lo, st);
    h->t_hi = th;
    h->t_lo = tl;
    h->ws_M = newM;
    clear_call_maps(h);  // maps over t must be rebuilt
  }
  return LL_OK;
}

// Grow the FP8-operand path's buffers (token exponents, e4m3 codes of x)
// to `M` rows (stream-ordered).
int f8_cluster_count(const ll_layer* h);

int ensure_f8_workspace(ll_layer* h, int M, cudaStream_t st) {
  if (!h->f8_part) {
    // Two partial-tile slots per CTA pair.
    const size_t bytes = static_cast<size_t>(f8_cluster_count(h)) * 2 * 2 * llk::kF8PartFloats * sizeof(float);
    if (cudaMallocAsync(reinterpret_cast<void**>(&h->f8_part), bytes, st) != cudaSuccess) {
      cudaGetLastError();
      h->f8_part = nullptr;
      return LL_ERR_OOM;
    }
  }
  if (M <= h->ws8_M) return LL_OK;
  int newM = std::max(M, h->ws8_M * 3 / 2);
  newM = (newM + 255) / 256 * 256;
  int *e = nullptr, *cnt = nullptr;
  uint8_t *a = nullptr, *b = nullptr;
  const size_t bytes = static_cast<size_t>(newM) * h->K;
  const size_t ncnt = static_cast<size_t>(newM / 256) * ((h->N + 255) / 256) * 8;
  if (cudaMallocAsync(reinterpret_cast<void**>(&e), sizeof(int) * newM, st) != cudaSuccess ||
      cudaMallocAsync(reinterpret_cast<void**>(&a), bytes, st) != cudaSuccess ||
      cudaMallocAsync(reinterpret_cast<void**>(&b), bytes, st) != cudaSuccess ||
      cudaMallocAsync(reinterpret_cast<void**>(&cnt), sizeof(int) * ncnt, st) != cudaSuccess ||
      cudaMemsetAsync(cnt, 0, sizeof(int) * ncnt, st) != cudaSuccess) {
    cudaGetLastError();
    if (e) cudaFreeAsync(e, st);
    if (a) cudaFreeAsync(a, st);
    if (b) cudaFreeAsync(b, st);
    if (cnt) cudaFreeAsync(cnt, st);
    return LL_ERR_OOM;
  }
  if (h->e_tok) cudaFreeAsync(h->e_tok, st);
  if (h->xh) cudaFreeAsync(h->xh, st);
  if (h->xl) cudaFreeAsync(h->xl, st);
  if (h->f8_cnt) cudaFreeAsync(h->f8_cnt, st);
  h->e_tok = e;
  h->xh = a;
  h->xl = b;
  h->f8_cnt = cnt;
  h->f8_cnt_n = ncnt;
  h->ws8_M = newM;
  clear_call_maps(h);  // maps over the codes must be rebuilt
  return LL_OK;
}

enum Path { PATH_SMALL, PATH_TC1, PATH_TC2, PATH_STREAM, PATH_F8, PATH_F8S, PATH_GEMV };

bool is_geglu(const ll_layer* h) { return h->epilogue == LL_EPILOGUE_GEGLU_TANH; }
// Columns of y: N, or N / 2 when the epilogue is GEGLU.
int out_features(const ll_layer* h) { return is_geglu(h) ? h->N / 2 : h->N; }
// Activation code of the kernels' epilogues (epi_act).
int act_code(const ll_layer* h) {
  return h->epilogue == LL_EPILOGUE_GELU_TANH    ? llk::kActGelu
         : h->epilogue == LL_EPILOGUE_GEGLU_TANH ? llk::kActGeglu
                                                 : llk::kActNone;
}

// Where the two-term FP8-operand kernel beats the one-CTA exact-widening
// kernel for M > 256.  Its split of x costs 2MK bytes each way against a
// GEMM of 2MNK flops, so it wins on wide layers.  Measured forward times on
// B200 (us, exact-widening / two-term): N = 4K: 3630 x 2048 -> 8192 122 / 101,
// 1024 x 4096 -> 16384 122 / 108, 16384 x 4096 -> 16384 1727 / 1470;
// N = K: 4096 x 4096 -> 4096 124 / 118, 16384 x 4096 -> 4096 450 / 415,
// 1024 x 4096 -> 4096 40 / 63, 3630 x 2048 -> 2048 42 / 54;
// N = K / 4: 3630 x 8192 -> 2048 118 / 169, 9800 x 16384 -> 4096 1071 / 1112.
bool fp8_split_wins(int N, int K, int M) { return N >= 2 * K || (N >= K && M >= 4096); }

constexpr int kStreamMaxM = 64;
bool gemv_fits(const ll_layer* h, int M) {
  return M <= llk::kGvMaxM && llk::gv_smem_bytes(M, h->K) <= 227u * 1024u;
}
constexpr int kF8sLrBudget = 20;  // SMs for the down-projection beside the FP8-operand streaming kernel
constexpr int kPairMaxM = 256;

Path choose_path(const ll_layer* h, int M) {
  // The FP8-operand variants: the streaming kernel up to 64 tokens (not with
  // GEGLU, whose value and gate rows sit in different 128-feature tiles
  // there), the CTA-pair kernel above.
  if (h->variant == LL_VARIANT_FP8_SPLIT || h->variant == LL_VARIANT_FP8_ACT)
    return M <= kStreamMaxM && !is_geglu(h) ? PATH_F8S : PATH_F8;
  // GEGLU pairs value and gate features inside a thread: the FP8-operand
  // kernel holds a token's features in one thread; the others do not.
  if (is_geglu(h) && h->variant == LL_VARIANT_AUTO) return PATH_F8;
  // CUDA-core GEMV: M <= 4 with x fitting in shared memory beside the ring.
  if (h->variant == LL_VARIANT_GEMV) return gemv_fits(h, M) ? PATH_GEMV : PATH_SMALL;
  if (h->variant == LL_VARIANT_TC) return PATH_TC1;
  if (h->variant == LL_VARIANT_TC_PAIR) return PATH_TC2;
  if (h->variant == LL_VARIANT_SMALL) return PATH_SMALL;
  if (h->variant == LL_VARIANT_STREAM) return M <= kStreamMaxM ? PATH_STREAM : PATH_SMALL;
  // One token: the CUDA-core GEMV (measured at K = 4096, N = 16384,
  // r = 512: 29.7 against 31.8 us; from two tokens on the streaming kernel
  // leads, 31.7 against 33.8).
  if (M == 1 && gemv_fits(h, M)) return PATH_GEMV;
  if (M <= kStreamMaxM) return PATH_STREAM;
  // Measured on the K = 4096, N = 16384 family: the CTA-pair kernel with
  // its narrow tiles beats the 128 x 128 and one-CTA kernels up to 256
  // tokens; above, the one-CTA kernel with its joint plan, except where the
  // FP8-operand kernel is faster.
  if (M <= kPairMaxM) return PATH_TC2;
  return fp8_split_wins(h->N, h->K, M) ? PATH_F8 : PATH_TC1;
}

// CTAs of the streaming kernel: one per 128-feature tile, at most one per SM.
int stream_ctas(const ll_layer* h) { return std::min((h->N + 127) / 128, h->num_sms); }

// Joint plan of the single-CTA fused kernel and the down-projection beside
// it.  The down-projection's CTAs hold their SMs until t is written, so the
// fused kernel's CTAs on those SMs start late and (taking tiles from a
// shared counter) take fewer tiles.  The plan picks the tile width (a
// multiple of 32 from 128 to 256) and the number of K splits of the
// down-projection that minimise a model of the finishing time: tiles of
// equal duration handed out greedily to the SMs free at time 0 and to the
// down-projection's SMs once it ends.  The model's rates are fitted to
// forward times measured on B200 (they rank plans; they are not a
// prediction of the time).
double tc_finish_us(long long tiles, int sms, int late, double t_tile, double t_lr) {
  const int early = sms - late;
  // A tile's low-rank step needs t: early tiles cannot end before it is there.
  const double d0 = std::max(0.0, t_lr + 1.0 - t_tile);
  long long done = 0;
  long long ke = 0, kl = 0;
  for (;;) {
    const double se = early > 0 ? d0 + ke * t_tile : 1e30;
    const double sl = late > 0 ? t_lr + kl * t_tile : 1e30;
    double s;
    if (se <= sl) {
      done += early;
      s = se;
      ++ke;
    } else {
      done += late;
      s = sl;
      ++kl;
    }
    if (done >= tiles) return s + t_tile;
  }
}

// The finishing-time model over `slots` places for tiles of `feat`
// features (SMs for the one-CTA kernel, clusters for the CTA pairs; one
// down-projection CTA takes 1 / `sms_per_slot` of a place), tile widths
// from 256 down to `bt_min` tokens.
TcChoice plan_joint(const ll_layer* h, int M, int feat, int slots, int sms_per_slot, int bt_min) {
  constexpr double kStageNsPerToken = 2.8;  // per 2-K-step stage and (bt + 32) tokens
  constexpr double kTileFixedUs = 2.5;      // pipeline fill + epilogue per tile
  constexpr double kLrFixedUs = 3.5;        // down-projection launch, first loads, reduction
  constexpr double kLrCtaGBs = 70.0;        // x read rate of one down-projection CTA
  constexpr double kLrMaxGBs = 5500.0;      // and of all of them together
  const int nK = (h->K + llk::kBK - 1) / llk::kBK;
  const int nS = (nK + 1) / 2;
  const int n_ftiles = (h->N + feat - 1) / feat;
  const int m_tiles = (M + 127) / 128;
  const int rc = std::min(std::max(h->r_pad, 32), 256);
  const int r_chunks = h->r_pad > 0 ? (h->r_pad + rc - 1) / rc : 0;
  const double x_mb = 2.0 * M * h->K * r_chunks / 1e6;
  TcChoice best{256, 1};
  double best_t = -1;
  for (int bt = 256; bt >= bt_min; bt -= 32) {
    const long long tiles = static_cast<long long>(n_ftiles) * ((M + bt - 1) / bt);
    const double t_tile = kTileFixedUs + 0.3 * h->r_pad / 32 + nS * (bt + 32) * kStageNsPerToken * 1e-3;
    const int ks_max = h->r_pad > 0 ? std::min(nK, llk::kLrMaxSplit) : 1;
    for (int ks = 1; ks <= ks_max; ++ks) {
      const int lr_ctas = h->r_pad > 0 ? m_tiles * r_chunks * ks : 0;
      if (ks > 1 && lr_ctas > h->num_sms) break;
      const int late = std::min((lr_ctas + sms_per_slot - 1) / sms_per_slot, slots);
      const double t_lr =
          h->r_pad > 0 ? kLrFixedUs + x_mb / std::min(std::max(lr_ctas, 1) * kLrCtaGBs, kLrMaxGBs) * 1e3 : 0.0;
      const double t = tc_finish_us(tiles, slots, late, t_tile, t_lr);
      // A wider tile or fewer down-projection CTAs unless the model gains
      // more than 1 %.
      if (best_t < 0 || t < best_t * 0.99) {
        best_t = t;
        best = TcChoice{bt, ks};
      }
    }
  }
  return best;
}

TcChoice plan_tc1(const ll_layer* h, int M) {
  if (h->tcp_M != M) {
    h->tcp = plan_joint(h, M, 128, h->num_sms, 1, 128);
    h->tcp_M = M;
  }
  return h->tcp;
}

int tc_tile_tokens(const ll_layer* h, int M) { return plan_tc1(h, M).bt; }

int pair_cluster_count(const ll_layer* h);

// The same joint plan for the CTA-pair kernel: tiles of 256 features over
// the co-resident clusters, tile widths down to 32 tokens (small M), and a
// down-projection CTA taking half a cluster's SMs.
TcChoice plan_tc2(const ll_layer* h, int M) {
  if (h->tcp2_M != M) {
    h->tcp2 = plan_joint(h, M, 256, pair_cluster_count(h), 2, 32);
    h->tcp2_M = M;
  }
  return h->tcp2;
}

int tc2_tile_tokens(ll_layer* h, int M) { return plan_tc2(h, M).bt; }

struct LrPlan {
  int rc;            // column block of t per CTA (B box height)
  int tmem_cols;     // power of two >= rc
  int ksplit, kb_per_split, m_tiles, r_chunks;
};

LrPlan plan_lowrank(const ll_layer* h, int M) {
  LrPlan p{};
  const int nK = (h->K + llk::kBK - 1) / llk::kBK;
  p.m_tiles = (M + 127) / 128;
  if (h->r_pad == 0) {
    p.rc = 32;
    p.tmem_cols = 32;
    p.ksplit = 1;
    p.kb_per_split = nK;
    p.r_chunks = 0;
    return p;
  }
  p.rc = std::min(h->r_pad, 256);
  const Path path = choose_path(h, M);
  const bool fused_large = path != PATH_SMALL;
  // Few token tiles: narrower column blocks so more CTAs share the read of B.
  if (!fused_large && p.rc > 128 && p.m_tiles * ((h->r_pad + 127) / 128) <= h->num_sms / 2) p.rc = 128;
  p.r_chunks = (h->r_pad + p.rc - 1) / p.rc;
  p.tmem_cols = next_pow2_ge32(p.rc);
  const int ctas = p.m_tiles * p.r_chunks;
  // The down-projection runs beside the fused kernels: as many splits as
  // the joint plans give next to the single-CTA and CTA-pair kernels, and
  // the SMs the streaming kernel's tiles leave free.  The other kernels
  // wait for it, so it takes all SMs.
  int budget = h->num_sms;
  if (path == PATH_STREAM) budget = std::max(1, h->num_sms - stream_ctas(h));
  // Beside the FP8-operand kernel, whose tiles need t only at their end:
  // half of the SMs.
  if (path == PATH_F8) budget = std::max(1, h->num_sms / 2);
  // Beside the FP8-operand streaming kernel: about as many SMs as the
  // exact streaming kernel leaves free at the small-batch shape.
  if (path == PATH_F8S) budget = kF8sLrBudget;
  int ks = std::max(1, budget / ctas);
  ks = std::min(std::min(ks, nK), llk::kLrMaxSplit);
  if (path == PATH_TC1 && M > 128) ks = plan_tc1(h, M).ks;
  if (path == PATH_TC2) ks = plan_tc2(h, M).ks;
  p.kb_per_split = (nK + ks - 1) / ks;
  p.ksplit = (nK + p.kb_per_split - 1) / p.kb_per_split;
  return p;
}

// Launches the down-projection; its K splits form one cluster per tile.
// With lpp.wait_prior it is a programmatic dependent of the kernel before.
cudaError_t launch_lrdown(const llk::LrDownParams& lpp, const LrPlan& lp, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(lp.m_tiles, lp.r_chunks, lp.ksplit);
  cfg.blockDim = dim3(llk::kLrThreads);
  cfg.dynamicSmemBytes = llk::lr_smem_bytes(lp.rc);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (lp.ksplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = static_cast<unsigned>(lp.ksplit);
    ++na;
  }
  if (lpp.wait_prior) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, llk::ll_lrdown_kernel, lpp);
}

bool build_call_maps_uncached(ll_layer* h, const void* x, void* y, int M, bool f8);

// The descriptor set of (x, y, M): the current one, a cached one, or a new
// one (kept in the cache, oldest entry replaced).
bool build_call_maps(ll_layer* h, const void* x, void* y, int M, bool f8) {
  auto match = [&](const CallMaps& c) { return c.c_x == x && c.c_yptr == y && c.c_M == M && (!f8 || c.c_f8); };
  if (match(h->cm)) return true;
  for (const CallMaps& c : h->cm_cache)
    if (match(c)) {
      h->cm = c;
      return true;
    }
  if (!build_call_maps_uncached(h, x, y, M, f8)) return false;
  h->cm_cache[h->cm_next] = h->cm;
  h->cm_next = (h->cm_next + 1) % kMapCache;
  return true;
}

bool build_call_maps_uncached(ll_layer* h, const void* x, void* y, int M, bool f8) {
  using namespace llk;
  bool ok = true;
  if (f8) {
    constexpr CUtensorMapDataType kU8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    ok &= make_map(&h->cm.c_xh, h->xh, kU8, M, h->K, h->K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&h->cm.c_xl, h->xl, kU8, M, h->K, h->K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&h->cm.c_y64, y, kBF16, M, out_features(h), 2ull * out_features(h), 32, 32,
                   CU_TENSOR_MAP_SWIZZLE_64B);
    if (M <= kStreamMaxM) {
      const uint32_t Mt = static_cast<uint32_t>((M + 15) / 16 * 16);
      ok &= make_map(&h->cm.c_xhs, h->xh, kU8, M, h->K, h->K, 128, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= make_map(&h->cm.c_xls, h->xl, kU8, M, h->K, h->K, 128, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (h->r_pad > 0) {
      ok &= make_map(&h->cm.c_thi32, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
      ok &= make_map(&h->cm.c_tlo32, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
    }
  }
  h->cm.c_f8 = f8;
  ok &= make_map(&h->cm.c_x128, x, kBF16, M, h->K, 2ull * h->K, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&h->cm.c_x256, x, kBF16, M, h->K, 2ull * h->K, kBK, 256, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&h->cm.c_y, y, kBF16, M, h->N, 2ull * h->N, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (M > 128) {
    const int bt = tc_tile_tokens(h, M);
    h->cm.c_bt = bt;
    ok &= make_map(&h->cm.c_xbt, x, kBF16, M, h->K, 2ull * h->K, kBK, bt, CU_TENSOR_MAP_SWIZZLE_128B);
    if (h->r_pad > 0) {
      const CUtensorMapSwizzle sw = h->klr == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
      ok &= make_map(&h->cm.c_thibt, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, bt, sw);
      ok &= make_map(&h->cm.c_tlobt, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, bt, sw);
    }
  }
  {
    // CTA-pair kernel maps (every M: any variant may be chosen later).
    const int bt2 = tc2_tile_tokens(h, M);
    const uint32_t hb = static_cast<uint32_t>(bt2 / 2);
    h->cm.c_bt2 = bt2;
    if (h->K % 64 == 0)
      ok &= make_map3(&h->cm.c_x2p, x, kBF16, 64, M, h->K / 64, 2ull * h->K, 128, 64, hb, 2, CU_TENSOR_MAP_SWIZZLE_128B);
    else
      ok &= make_map(&h->cm.c_x2p, x, kBF16, M, h->K, 2ull * h->K, kBK, hb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (h->r_pad > 0) {
      const CUtensorMapSwizzle sw = h->klr == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
      ok &= make_map(&h->cm.c_thip, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, hb, sw);
      ok &= make_map(&h->cm.c_tlop, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, hb, sw);
    }
  }
  if (M <= kStreamMaxM) {
    const uint32_t Mt = static_cast<uint32_t>((M + 15) / 16 * 16);
    if (h->K % 64 == 0)
      ok &= make_map3(&h->cm.c_xs, x, kBF16, 64, M, h->K / 64, 2ull * h->K, 128, 64, Mt, 4, CU_TENSOR_MAP_SWIZZLE_128B);
    else
      ok &= make_map(&h->cm.c_xs, x, kBF16, M, h->K, 2ull * h->K, kBK, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
    if (h->r_pad > 0) {
      ok &= make_map(&h->cm.c_this, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, kBK, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= make_map(&h->cm.c_tlos, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, kBK, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
    }
  }
  if (h->r_pad > 0) {
    const CUtensorMapSwizzle sw = h->klr == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    ok &= make_map(&h->cm.c_thi128, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&h->cm.c_tlo128, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&h->cm.c_thi256, h->t_hi, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, 256, sw);
    ok &= make_map(&h->cm.c_tlo256, h->t_lo, kBF16, M, h->r_pad, 2ull * h->r_pad, h->klr, 256, sw);
  }
  if (!ok) {
    h->cm.c_M = -1;
    return false;
  }
  h->cm.c_x = x;
  h->cm.c_yptr = y;
  h->cm.c_M = M;
  return true;
}

// Data-parallel waves of the FP8-operand kernel before its stream-K tiles.
// By default every tile is whole and taken from the counter.  Measured on
// B200, spreading the last partial wave stream-K over all pairs does not
// pay: the attention projection (120 tiles on 74 pairs) took 77 us against
// 56 us whole, its split tiles' fp32 partials costing 4 to 13 us of memory
// latency per pair in the epilogue.  LL_FP8_STREAMK=1 in the environment
// turns the stream-K tail on (the last partial wave, merged with the whole
// wave before it when it is shorter than half a wave), for measurements.
int f8_dp_waves(int tiles, int clusters) {
  static const int sk = [] {
    const char* e = std::getenv("LL_FP8_STREAMK");
    return e && e[0] == '1' ? 1 : 0;
  }();
  const int whole = (tiles + clusters - 1) / clusters;
  if (!sk) return whole;
  int D = tiles / clusters;
  const int S = tiles - D * clusters;
  if (S > 0 && D > 0 && 2 * S < clusters) --D;
  return D;
}

// Co-resident clusters of the FP8-operand kernel (asked once per layer).
int f8_cluster_count(const ll_layer* h) {
  if (h->f8_clusters > 0) return h->f8_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->num_sms);
  cfg.blockDim = dim3(llk::kF8Threads);
  cfg.dynamicSmemBytes = llk::f8_smem_bytes();
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel_f8(llk::kActNone), &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = h->num_sms / 2;
  }
  h->f8_clusters = std::min(n, h->num_sms / 2);
  return h->f8_clusters;
}

int pair_cluster_count(const ll_layer* h) {
  if (h->pair_clusters > 0) return h->pair_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->num_sms);
  cfg.blockDim = dim3(llk::kT2Threads);
  cfg.dynamicSmemBytes = llk::tc2_smem_bytes();
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel_tc2(llk::kActNone), &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = h->num_sms / 2;
  }
  h->pair_clusters = std::min(n, h->num_sms / 2);
  return h->pair_clusters;
}

// M <= 4 on CUDA cores: t = x B^T (fp32) and the fused GEMV, a programmatic
// dependent of it that waits only before its low-rank part.
int forward_gemv(ll_layer* h, const void* x, void* y, int M, cudaStream_t st) {
  using namespace llk;
  if (h->r_pad > 0 && !h->t32) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&h->t32), sizeof(float) * kGvMaxM * h->r_pad, st) != cudaSuccess) {
      cudaGetLastError();
      h->t32 = nullptr;
      return LL_ERR_OOM;
    }
  }
  int launches = 0;
  const bool prof = h->profiling != 0;
  h->prof_valid = 0;
  if (prof) {
    for (cudaEvent_t& e : h->ev)
      if (!e && cudaEventCreate(&e) != cudaSuccess) return LL_ERR_CUDA;
    cudaEventRecord(h->ev[0], st);
  }
  if (h->r_pad > 0) {
    const int grid = std::max(1, std::min(h->num_sms, (h->r_pad + kGvWarps - 1) / kGvWarps));
    kernel_gemv_t(M)<<<grid, kGvThreads, static_cast<size_t>(M) * h->K * 2, st>>>(
        static_cast<const uint16_t*>(x), h->B, h->t32, h->K, h->r_pad);
    h->names[launches++] = "ll_gemv_t_kernel";
    if (prof) cudaEventRecord(h->ev[launches], st);
    if (cudaGetLastError() != cudaSuccess) return LL_ERR_CUDA;
  }
  GemvParams gp;
  gp.x = static_cast<const uint16_t*>(x);
  gp.q = h->Q;
  gp.a = h->A;
  gp.t = h->t32;
  gp.scale = h->scale;
  gp.bias = h->has_bias ? h->bias : nullptr;
  gp.y = static_cast<uint16_t*>(y);
  gp.M = M;
  gp.N = h->N;
  gp.K = h->K;
  gp.r_pad = h->r_pad;
  const bool overlap = h->r_pad > 0 && !prof;
  gp.t_from_primary = overlap ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.gridDim = dim3(h->num_sms);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = gv_smem_bytes(M, h->K);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kernel_gemv(M, act_code(h)), gp) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  h->names[launches++] = "ll_gemv_kernel";
  if (prof) {
    cudaEventRecord(h->ev[launches], st);
    h->prof_valid = 1;
  }
  h->last_launches = launches;
  return LL_OK;
}

int forward_device(ll_layer* h, const void* x, void* y, int M, cudaStream_t st) {
  using namespace llk;
  h->last_launches = 0;
  const Path path = choose_path(h, M);
  if (is_geglu(h) && path != PATH_F8) return LL_ERR_UNSUPPORTED;
  if (path == PATH_GEMV) return forward_gemv(h, x, y, M, st);
  const bool f8 = path == PATH_F8 || path == PATH_F8S;
  const LrPlan lp = plan_lowrank(h, M);
  int rc = ensure_workspace(h, M, st);
  if (rc != LL_OK) return rc;
  if (f8) {
    rc = ensure_f8_workspace(h, M, st);
    if (rc != LL_OK) return rc;
  }
  if (!build_call_maps(h, x, y, M, f8)) return LL_ERR_CUDA;
  const Watch watch{h->status, h->timeout_ns};
  int launches = 0;
  const bool prof = h->profiling != 0;
  h->prof_valid = 0;
  if (prof) {
    for (cudaEvent_t& e : h->ev)
      if (!e && cudaEventCreate(&e) != cudaSuccess) return LL_ERR_CUDA;
    cudaEventRecord(h->ev[0], st);
  }

  const int f8_terms = h->variant == LL_VARIANT_FP8_ACT ? 1 : 2;
  if (f8) {
    // Per-token exponents and e4m3 codes of x; the down-projection and the
    // FP8-operand kernel below both read them.
    const int blocks = std::max(1, std::min((M + 7) / 8, h->num_sms * 8));
    ll_xsplit_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(x), M, h->K, f8_terms, h->e_tok, h->xh,
                                            h->xl);
    h->names[launches++] = "ll_xsplit_kernel";
    if (prof) cudaEventRecord(h->ev[launches], st);
    if (cudaGetLastError() != cudaSuccess) return LL_ERR_CUDA;
  }

  if (h->r_pad > 0) {
    if (lp.rc != h->b_box) {
      if (!make_map(&h->tm_b, h->B, kBF16, h->r_pad, h->K, 2ull * h->K, kBK, lp.rc, CU_TENSOR_MAP_SWIZZLE_128B))
        return LL_ERR_CUDA;
      h->b_box = lp.rc;
    }
    LrDownParams lpp;
    lpp.tm_x = h->cm.c_x128;
    lpp.tm_b = h->tm_b;
    lpp.t_hi = h->t_hi;
    lpp.t_lo = h->t_lo;
    lpp.M = M;
    lpp.K = h->K;
    lpp.r_pad = h->r_pad;
    lpp.rc = lp.rc;
    lpp.tmem_cols = lp.tmem_cols;
    lpp.ksplit = lp.ksplit;
    lpp.kb_per_split = lp.kb_per_split;
    lpp.e_tok = f8 ? h->e_tok : nullptr;
    // Beside the split of x, which writes the token exponents it reads.
    lpp.wait_prior = f8 && !prof ? 1 : 0;
    lpp.watch = watch;
    const cudaError_t lerr = launch_lrdown(lpp, lp, st);
    h->names[launches++] = "ll_lrdown_kernel";
    if (prof) cudaEventRecord(h->ev[launches], st);
    if (lerr != cudaSuccess) {
      cudaGetLastError();
      return LL_ERR_CUDA;
    }
  }

  // Programmatic overlap with the kernel that produces t.
  const bool overlap = h->r_pad > 0 && !prof;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  cudaError_t err;
  if (path == PATH_F8) {
    F8Params fp;
    fp.tm_xh = h->cm.c_xh;
    fp.tm_xl = h->cm.c_xl;
    fp.tm_q = h->tm_q128;
    fp.tm_ahi = h->tm_ahi32;
    fp.tm_alo = h->tm_alo32;
    fp.tm_thi = h->r_pad > 0 ? h->cm.c_thi32 : h->cm.c_xh;  // unused when r_pad == 0
    fp.tm_tlo = h->r_pad > 0 ? h->cm.c_tlo32 : h->cm.c_xh;
    fp.tm_y = h->cm.c_y64;
    fp.e_tok = h->e_tok;
    fp.scale = h->scale_eff;
    fp.bias = h->has_bias ? h->bias : nullptr;
    fp.part = h->f8_part;
    fp.cnt = h->f8_cnt;
    fp.sched = h->sched;
    fp.M = M;
    fp.N = h->N;
    fp.K = h->K;
    fp.r_pad = h->r_pad;
    fp.terms = f8_terms;
    fp.n_ttiles = (M + 255) / 256;
    fp.n_ftiles = (h->N + 255) / 256;
    fp.lr_from_primary = overlap ? 1 : 0;
    fp.withhold = h->withhold;
    fp.watch = watch;
    // Stream-K over (tile, 128-wide K step) units: one equal range per pair.
    const long long units = static_cast<long long>(fp.n_ttiles) * fp.n_ftiles * ((h->K + 127) / 128);
    const int clusters = static_cast<int>(std::max(1LL, std::min<long long>(f8_cluster_count(h), units)));
    fp.clusters = clusters;
    fp.dp_waves = is_geglu(h) ? (fp.n_ttiles * fp.n_ftiles + clusters - 1) / clusters
                              : f8_dp_waves(fp.n_ttiles * fp.n_ftiles, clusters);
    if (fp.dp_waves * clusters < fp.n_ttiles * fp.n_ftiles) {
      // Stream-K splits the last wave evenly over all pairs, so they must
      // all start together: no overlap with the down-projection, which
      // would hold some SMs at the start.
      cfg.numAttrs = 0;
      fp.lr_from_primary = 0;
    }
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(kF8Threads);
    cfg.dynamicSmemBytes = f8_smem_bytes();
    err = cudaLaunchKernelEx(&cfg, kernel_f8(act_code(h)), fp);
    h->names[launches] = "ll_f8_kernel";
  } else if (path == PATH_F8S) {
    F8sParams fs;
    fs.tm_q = h->tm_q128;
    fs.tm_xh = h->cm.c_xhs;
    fs.tm_xl = h->cm.c_xls;
    fs.tm_a = h->r_pad > 0 ? h->tm_a : h->tm_q128;  // unused when r_pad == 0
    fs.tm_thi = h->r_pad > 0 ? h->cm.c_this : h->cm.c_xhs;
    fs.tm_tlo = h->r_pad > 0 ? h->cm.c_tlos : h->cm.c_xhs;
    fs.e_tok = h->e_tok;
    fs.scale = h->scale;
    fs.bias = h->has_bias ? h->bias : nullptr;
    fs.y = static_cast<uint16_t*>(y);
    fs.part = h->f8_part;
    fs.cnt = h->f8_cnt;
    fs.M = M;
    fs.N = h->N;
    fs.K = h->K;
    fs.r_pad = h->r_pad;
    fs.Mt = (M + 15) / 16 * 16;
    fs.terms = f8_terms;
    fs.n_ftiles = (h->N + 127) / 128;
    // One CTA per SM that the down-projection leaves free; at most one per unit.
    const int lr_ctas = h->r_pad > 0 ? lp.m_tiles * lp.r_chunks * lp.ksplit : 0;
    const long long units =
        static_cast<long long>(fs.n_ftiles) * ((h->K + 127) / 128 + (h->r_pad + 63) / 64);
    fs.ctas = static_cast<int>(std::max(1LL, std::min<long long>(std::max(1, h->num_sms - lr_ctas), units)));
    fs.w_stages = ss_w_stages(fs.Mt);
    fs.lr_from_primary = overlap ? 1 : 0;
    fs.withhold = h->withhold;
    fs.watch = watch;
    cfg.gridDim = dim3(fs.ctas);
    cfg.blockDim = dim3(kSsThreads);
    cfg.dynamicSmemBytes = ss_smem_bytes(fs.Mt);
    err = cudaLaunchKernelEx(&cfg, kernel_f8s(act_code(h)), fs);
    h->names[launches] = "ll_f8_stream_kernel";
  } else if (path == PATH_STREAM) {
    StreamParams sp;
    const bool dims3 = h->K % 64 == 0;
    sp.tm_x = h->cm.c_xs;
    sp.tm_q = dims3 ? h->tm_q3 : h->tm_q;
    sp.tm_a = h->tm_a;
    sp.tm_thi = h->cm.c_this;
    sp.tm_tlo = h->cm.c_tlos;
    sp.scale = h->scale;
    sp.bias = h->has_bias ? h->bias : nullptr;
    sp.y = static_cast<uint16_t*>(y);
    sp.M = M;
    sp.N = h->N;
    sp.K = h->K;
    sp.r_pad = h->r_pad;
    sp.Mt = (M + 15) / 16 * 16;
    sp.n_ftiles = (h->N + 127) / 128;
    sp.dims3 = dims3 ? 1 : 0;
    sp.lr_from_primary = overlap ? 1 : 0;
    sp.withhold = h->withhold;
    sp.watch = watch;
    cfg.gridDim = dim3(stream_ctas(h));
    cfg.blockDim = dim3(kStThreads);
    cfg.dynamicSmemBytes = st_smem_bytes(sp.Mt);
    err = cudaLaunchKernelEx(&cfg, kernel_stream(act_code(h)), sp);
    h->names[launches] = "ll_stream_kernel";
  } else if (path == PATH_TC2) {
    Tc2Params tp;
    tp.dims3 = h->K % 64 == 0 ? 1 : 0;
    tp.tm_x = h->cm.c_x2p;
    tp.tm_q = tp.dims3 ? h->tm_q3b2 : h->tm_qf;
    tp.tm_ahi = h->tm_ahi;
    tp.tm_alo = h->tm_alo;
    tp.tm_thi = h->cm.c_thip;
    tp.tm_tlo = h->cm.c_tlop;
    tp.tm_y = h->cm.c_y;
    tp.scale = h->scale_eff;
    tp.bias = h->has_bias ? h->bias : nullptr;
    tp.M = M;
    tp.N = h->N;
    tp.K = h->K;
    tp.r_pad = h->r_pad;
    tp.klr = h->klr;
    tp.bt = h->cm.c_bt2;
    tp.n_fpairs = (h->N + 255) / 256;
    tp.n_ttiles = (M + tp.bt - 1) / tp.bt;
    tp.sched = h->sched;
    const int tiles = tp.n_fpairs * tp.n_ttiles;
    const int clusters = std::max(1, std::min(pair_cluster_count(h), tiles));
    tp.lr_from_primary = overlap ? 1 : 0;
    tp.withhold = h->withhold;
    tp.watch = watch;
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(kT2Threads);
    cfg.dynamicSmemBytes = tc2_smem_bytes();
    err = cudaLaunchKernelEx(&cfg, kernel_tc2(act_code(h)), tp);
    h->names[launches] = "ll_tc2_kernel";
  } else if (path == PATH_TC1) {
    TcParams tp;
    const bool large = M > 128;  // the per-call maps of bt rows exist for M > 128
    tp.bt = large ? h->cm.c_bt : 256;
    tp.tm_x = large ? h->cm.c_xbt : h->cm.c_x256;
    tp.q3 = h->K % 64 == 0 ? 1 : 0;
    tp.tm_q = tp.q3 ? h->tm_q3b2 : h->tm_qf;
    tp.tm_ahi = h->tm_ahi;
    tp.tm_alo = h->tm_alo;
    tp.tm_thi = large ? h->cm.c_thibt : h->cm.c_thi256;
    tp.tm_tlo = large ? h->cm.c_tlobt : h->cm.c_tlo256;
    tp.tm_y = h->cm.c_y;
    tp.scale = h->scale_eff;
    tp.bias = h->has_bias ? h->bias : nullptr;
    tp.sched = h->sched;
    tp.M = M;
    tp.N = h->N;
    tp.K = h->K;
    tp.r_pad = h->r_pad;
    tp.klr = h->klr;
    tp.n_ftiles = (h->N + 127) / 128;
    tp.n_ttiles = (M + tp.bt - 1) / tp.bt;
    tp.lr_from_primary = overlap ? 1 : 0;
    tp.withhold = h->withhold;
    tp.watch = watch;
    const int tiles = tp.n_ftiles * tp.n_ttiles;
    cfg.gridDim = dim3(std::min(tiles, h->num_sms));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = tc_smem_bytes();
    err = cudaLaunchKernelEx(&cfg, kernel_tc(act_code(h)), tp);
    h->names[launches] = "ll_tc_kernel";
  } else {
    MainParams mp;
    mp.tm_x = h->cm.c_x128;
    mp.tm_q = h->tm_q;
    mp.tm_a = h->tm_a;
    mp.tm_thi = h->cm.c_thi128;
    mp.tm_tlo = h->cm.c_tlo128;
    mp.tm_y = h->cm.c_y;
    mp.scale = h->scale;
    mp.bias = h->has_bias ? h->bias : nullptr;
    mp.M = M;
    mp.N = h->N;
    mp.K = h->K;
    mp.r_pad = h->r_pad;
    mp.n_ftiles = (h->N + 127) / 128;
    mp.n_ttiles = (M + 127) / 128;
    mp.lr_from_primary = overlap ? 1 : 0;
    mp.withhold = h->withhold;
    mp.watch = watch;
    const int tiles = mp.n_ftiles * mp.n_ttiles;
    cfg.gridDim = dim3(std::min(tiles, h->num_sms));
    cfg.blockDim = dim3(kMainThreads);
    cfg.dynamicSmemBytes = main_smem_bytes();
    err = cudaLaunchKernelEx(&cfg, kernel_main(act_code(h)), mp);
    h->names[launches] = "ll_main_kernel";
  }
  if (err != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  ++launches;
  if (prof) {
    cudaEventRecord(h->ev[launches], st);
    h->prof_valid = 1;
  }
  h->last_launches = launches;
  return LL_OK;
}

}  // namespace

extern "C" {

const char* ll_status_string(int code) {
  switch (code) {
    case LL_OK: return "ok";
    case LL_ERR_INVALID_ARG: return "invalid argument";
    case LL_ERR_UNSUPPORTED: return "unsupported configuration";
    case LL_ERR_NOT_READY: return "weights not set";
    case LL_ERR_NAN_CODE: return "residual holds an e4m3fn NaN code";
    case LL_ERR_OOM: return "device allocation failed";
    case LL_ERR_CUDA: return "CUDA call failed";
    case LL_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case LL_ERR_SCRATCH_LIMIT: return "request exceeds the static scratch of ll_forward_noalloc";
    default: return "unknown status";
  }
}

int ll_last_error(void) { return g_last_error; }

ll_handle ll_create(int N, int K, int r, int scale_mode) {
  g_last_error = LL_OK;
  if (N < 1 || K < 16 || r < 0 || (N % 8) != 0 || (K % 16) != 0 ||
      (scale_mode != LL_SCALE_PER_TENSOR && scale_mode != LL_SCALE_PER_ROW)) {
    fail(LL_ERR_INVALID_ARG);
    return nullptr;
  }
  if (r > 512) {
    fail(LL_ERR_UNSUPPORTED);
    return nullptr;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    fail(LL_ERR_CUDA);
    return nullptr;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    fail(LL_ERR_CUDA);
    return nullptr;
  }
  if (prop.major != 10 || prop.minor != 0) {  // built for sm_100a only
    fail(LL_ERR_UNSUPPORTED);
    return nullptr;
  }
  if (set_smem_attrs_once() != 0 || !encode_fn()) {
    fail(LL_ERR_CUDA);
    return nullptr;
  }
  ll_layer* h = new ll_layer();
  h->N = N;
  h->K = K;
  h->r = r;
  h->r_pad = (r + 31) / 32 * 32;
  h->klr = (h->r_pad % 64 == 0) ? 64 : 32;
  h->scale_mode = scale_mode;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  bool ok = true;
  const size_t nrp = static_cast<size_t>(N) * h->r_pad;
  ok &= cudaMalloc(&h->Q, static_cast<size_t>(N) * K) == cudaSuccess;
  ok &= cudaMalloc(&h->scale, sizeof(float) * N) == cudaSuccess;
  ok &= cudaMalloc(&h->scale_eff, sizeof(float) * N) == cudaSuccess;
  ok &= cudaMalloc(&h->bias, sizeof(uint16_t) * N) == cudaSuccess;
  ok &= cudaMalloc(&h->status, sizeof(int)) == cudaSuccess;
  ok &= cudaMalloc(&h->flags, 2 * sizeof(int)) == cudaSuccess;
  ok &= cudaMalloc(&h->sched, 2 * sizeof(int)) == cudaSuccess;
  if (h->r_pad > 0) {
    ok &= cudaMalloc(&h->A, sizeof(uint16_t) * nrp) == cudaSuccess;
    ok &= cudaMalloc(&h->Ahi, sizeof(uint16_t) * nrp) == cudaSuccess;
    ok &= cudaMalloc(&h->Alo, sizeof(uint16_t) * nrp) == cudaSuccess;
    ok &= cudaMalloc(&h->B, sizeof(uint16_t) * static_cast<size_t>(h->r_pad) * K) == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    free_layer_mem(h);
    delete h;
    fail(LL_ERR_OOM);
    return nullptr;
  }
  h->Qf = h->Q;
  cudaMemset(h->status, 0, sizeof(int));
  cudaMemset(h->sched, 0, 2 * sizeof(int));
  using namespace llk;
  ok &= make_map(&h->tm_q, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, kBK, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  h->tm_qf = h->tm_q;
  if (K % 64 == 0) {
    ok &= make_map3(&h->tm_q3, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 4,
                    CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= make_map3(&h->tm_q3b2, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 2,
                    CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (h->r_pad > 0) {
    const CUtensorMapSwizzle sw = h->klr == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    ok &= make_map(&h->tm_a, h->A, kBF16, N, h->r_pad, 2ull * h->r_pad, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&h->tm_ahi, h->Ahi, kBF16, N, h->r_pad, 2ull * h->r_pad, h->klr, 128, sw);
    ok &= make_map(&h->tm_alo, h->Alo, kBF16, N, h->r_pad, 2ull * h->r_pad, h->klr, 128, sw);
    ok &= make_map(&h->tm_ahi32, h->Ahi, kBF16, N, h->r_pad, 2ull * h->r_pad, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= make_map(&h->tm_alo32, h->Alo, kBF16, N, h->r_pad, 2ull * h->r_pad, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  ok &= make_map(&h->tm_q128, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_layer_mem(h);
    delete h;
    fail(LL_ERR_CUDA);
    return nullptr;
  }
  return h;
}

int ll_set_weights(ll_handle h, const void* A, const void* B, const void* Q, const float* scale,
                   const void* bias) {
  g_last_error = LL_OK;
  if (!h || !Q || !scale) return fail(LL_ERR_INVALID_ARG);
  if (h->r > 0 && (!A || !B)) return fail(LL_ERR_INVALID_ARG);
  if (!aligned(Q, 16) || !aligned(scale, 4) || (bias && !aligned(bias, 2)) ||
      (h->r > 0 && (!aligned(A, 16) || !aligned(B, 16))))
    return fail(LL_ERR_INVALID_ARG);
  if (!is_device_ptr(Q) || !is_device_ptr(scale) || (bias && !is_device_ptr(bias)) ||
      (h->r > 0 && (!is_device_ptr(A) || !is_device_ptr(B))))
    return fail(LL_ERR_INVALID_ARG);
  const int N = h->N, K = h->K, r = h->r, rp = h->r_pad;
  const int ns = h->scale_mode == LL_SCALE_PER_ROW ? N : 1;
  std::vector<float> hs(ns);
  if (cudaMemcpy(hs.data(), scale, sizeof(float) * ns, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  for (float v : hs)
    if (!std::isfinite(v)) return fail(LL_ERR_INVALID_ARG);
  std::vector<float> full(N), eff(N);
  bool any_zero = false;
  for (int n = 0; n < N; ++n) {
    full[n] = hs[h->scale_mode == LL_SCALE_PER_ROW ? original_row(n, N, is_geglu(h)) : 0];
    eff[n] = full[n] == 0.f ? 1.f : full[n];
    any_zero |= full[n] == 0.f;
  }
  // NaN-code scan of the residual before anything of the handle changes.
  if (cudaMemset(h->flags, 0, 2 * sizeof(int)) != cudaSuccess) return fail(LL_ERR_CUDA);
  const size_t nq = static_cast<size_t>(N) * K;
  llk::ll_nan_scan_kernel<<<std::max(1, std::min(h->num_sms * 8, static_cast<int>((nq / 16 + 255) / 256))), 256>>>(
      static_cast<const uint8_t*>(Q), nq, h->flags);
  int flag = 0;
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpy(&flag, h->flags, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  if (flag) return fail(LL_ERR_NAN_CODE);
  h->ready = false;
  bool ok = true;
  ok &= copy_rows(h->Q, K, Q, K, K, N, is_geglu(h));
  ok &= cudaMemcpy(h->scale, full.data(), sizeof(float) * N, cudaMemcpyHostToDevice) == cudaSuccess;
  ok &= cudaMemcpy(h->scale_eff, eff.data(), sizeof(float) * N, cudaMemcpyHostToDevice) == cudaSuccess;
  if (bias) {
    ok &= copy_rows(h->bias, sizeof(uint16_t), bias, sizeof(uint16_t), sizeof(uint16_t), N, is_geglu(h));
  } else {
    ok &= cudaMemset(h->bias, 0, sizeof(uint16_t) * N) == cudaSuccess;
  }
  h->has_bias = bias != nullptr;
  // Residual used by the fused large-M kernel: rows with zero scale cleared.
  if (any_zero) {
    if (h->Qf == h->Q) {
      ok &= cudaMalloc(&h->Qf, nq) == cudaSuccess;
      ok &= make_map(&h->tm_qf, h->Qf, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, llk::kBK, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B);
      ok &= make_map(&h->tm_q128, h->Qf, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
      if (K % 64 == 0) {
        ok &= make_map3(&h->tm_q3, h->Qf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 4,
                        CU_TENSOR_MAP_SWIZZLE_64B);
        ok &= make_map3(&h->tm_q3b2, h->Qf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 2,
                        CU_TENSOR_MAP_SWIZZLE_64B);
      }
    }
    if (ok) {
      llk::ll_zero_rows_kernel<<<h->num_sms * 8, 256>>>(h->Q, h->scale, h->Qf, N, K);
      ok &= cudaGetLastError() == cudaSuccess;
    }
  } else if (h->Qf != h->Q) {
    cudaFree(h->Qf);
    h->Qf = h->Q;
    h->tm_qf = h->tm_q;
    ok &= make_map(&h->tm_q128, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (K % 64 == 0) {
      ok &= make_map3(&h->tm_q3, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 4,
                      CU_TENSOR_MAP_SWIZZLE_64B);
      ok &= make_map3(&h->tm_q3b2, h->Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, N, K / 64, K, 64, 64, 128, 2,
                      CU_TENSOR_MAP_SWIZZLE_64B);
    }
  }
  if (rp > 0) {
    ok &= cudaMemset(h->A, 0, sizeof(uint16_t) * N * static_cast<size_t>(rp)) == cudaSuccess;
    ok &= cudaMemset(h->B, 0, sizeof(uint16_t) * static_cast<size_t>(rp) * K) == cudaSuccess;
    ok &= copy_rows(h->A, sizeof(uint16_t) * rp, A, sizeof(uint16_t) * r, sizeof(uint16_t) * r, N, is_geglu(h));
    ok &= cudaMemcpy(h->B, B, sizeof(uint16_t) * static_cast<size_t>(r) * K, cudaMemcpyDeviceToDevice) ==
          cudaSuccess;
    if (ok) {
      llk::ll_fold_prep_kernel<<<h->num_sms * 8, 256>>>(h->A, h->scale_eff, h->Ahi, h->Alo, N, rp,
                                                         h->flags + 1);
      ok &= cudaGetLastError() == cudaSuccess;
    }
  }
  ok &= cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  int range_flag = 0;
  if (rp > 0 && cudaMemcpy(&range_flag, h->flags + 1, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  if (range_flag) return fail(LL_ERR_UNSUPPORTED);  // |A / scale| outside [2^-100, 2^100]
  h->ready = true;
  return LL_OK;
}

int ll_forward(ll_handle h, const void* x, void* y, int M, void* stream) {
  g_last_error = LL_OK;
  if (!h) return fail(LL_ERR_INVALID_ARG);
  if (M < 0) return fail(LL_ERR_INVALID_ARG);
  if (!h->ready) return fail(LL_ERR_NOT_READY);
  if (M == 0) {
    h->last_launches = 0;
    return LL_OK;
  }
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return fail(LL_ERR_INVALID_ARG);
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  const size_t xs = static_cast<size_t>(M) * h->K * 2, ys = static_cast<size_t>(M) * out_features(h) * 2;
  if (xb < yb + ys && yb < xb + xs) return fail(LL_ERR_INVALID_ARG);
  int rc = forward_device(h, x, y, M, static_cast<cudaStream_t>(stream));
  return rc == LL_OK ? LL_OK : fail(rc);
}

int ll_forward_host(ll_handle h, const void* x_host, void* y_host, int M, void* stream) {
  g_last_error = LL_OK;
  if (!h) return fail(LL_ERR_INVALID_ARG);
  if (M < 0 || (M > 0 && (!x_host || !y_host))) return fail(LL_ERR_INVALID_ARG);
  if (!h->ready) return fail(LL_ERR_NOT_READY);
  if (M == 0) return LL_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t xrow = static_cast<size_t>(h->K) * 2, yrow = static_cast<size_t>(out_features(h)) * 2;
  const size_t xs = static_cast<size_t>(M) * xrow, ys = static_cast<size_t>(M) * yrow;
  if (!h->cin) {
    bool ok = cudaStreamCreateWithFlags(&h->cin, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->cout, cudaStreamNonBlocking) == cudaSuccess;
    for (cudaEvent_t& e : h->hev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return fail(LL_ERR_CUDA);
    }
  }
  if (xs > h->dx_bytes) {
    void* p = nullptr;
    if (cudaMallocAsync(&p, xs, st) != cudaSuccess) { cudaGetLastError(); return fail(LL_ERR_OOM); }
    if (h->dx) cudaFreeAsync(h->dx, st);
    h->dx = p;
    h->dx_bytes = xs;
  }
  if (ys > h->dy_bytes) {
    void* p = nullptr;
    if (cudaMallocAsync(&p, ys, st) != cudaSuccess) { cudaGetLastError(); return fail(LL_ERR_OOM); }
    if (h->dy) cudaFreeAsync(h->dy, st);
    h->dy = p;
    h->dy_bytes = ys;
  }
  // Chunks of whole 256-token tiles: the copy of chunk i + 1 into the
  // device, the forward of chunk i and the copy of chunk i - 1 out run at
  // the same time (the two copy directions on their own streams).  The
  // caller's stream waits for the last copy out, so synchronising it once
  // still covers the whole call.
  // Up to four chunks: the copies are the bound (tens of GB/s against the
  // forward's TB/s).  Eight chunks measured slower than four on the
  // attention projection (each copy and each forward has a fixed cost);
  // below 512 tokens one chunk (each chunk reads the weights again).
  const int n_chunks = M >= 2048 ? 4 : (M >= 512 ? 2 : 1);
  const int rows = (M + n_chunks * 256 - 1) / (n_chunks * 256) * 256;
  cudaEvent_t* ev_in = h->hev + 1;
  cudaEvent_t* ev_fwd = h->hev + 1 + 8;
  cudaEvent_t ev_done = h->hev[2 * 8 + 1];
  if (cudaEventRecord(h->hev[0], st) != cudaSuccess || cudaStreamWaitEvent(h->cin, h->hev[0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(h->cout, h->hev[0], 0) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  int n = 0;
  for (int m0 = 0; m0 < M; m0 += rows, ++n) {
    const int mi = std::min(rows, M - m0);
    if (cudaMemcpyAsync(static_cast<char*>(h->dx) + m0 * xrow, static_cast<const char*>(x_host) + m0 * xrow,
                        mi * xrow, cudaMemcpyHostToDevice, h->cin) != cudaSuccess ||
        cudaEventRecord(ev_in[n], h->cin) != cudaSuccess) {
      cudaGetLastError();
      return fail(LL_ERR_CUDA);
    }
  }
  n = 0;
  for (int m0 = 0; m0 < M; m0 += rows, ++n) {
    const int mi = std::min(rows, M - m0);
    if (cudaStreamWaitEvent(st, ev_in[n], 0) != cudaSuccess) {
      cudaGetLastError();
      return fail(LL_ERR_CUDA);
    }
    const int rc = forward_device(h, static_cast<char*>(h->dx) + m0 * xrow, static_cast<char*>(h->dy) + m0 * yrow,
                                  mi, st);
    if (rc != LL_OK) return fail(rc);
    if (cudaEventRecord(ev_fwd[n], st) != cudaSuccess || cudaStreamWaitEvent(h->cout, ev_fwd[n], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<char*>(y_host) + m0 * yrow, static_cast<char*>(h->dy) + m0 * yrow, mi * yrow,
                        cudaMemcpyDeviceToHost, h->cout) != cudaSuccess) {
      cudaGetLastError();
      return fail(LL_ERR_CUDA);
    }
  }
  if (cudaEventRecord(ev_done, h->cout) != cudaSuccess || cudaStreamWaitEvent(st, ev_done, 0) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  return LL_OK;
}

int ll_reserve(ll_handle h, int max_M) {
  g_last_error = LL_OK;
  if (!h || max_M < 0) return fail(LL_ERR_INVALID_ARG);
  int rc = ensure_workspace(h, max_M, 0);
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    rc = LL_ERR_CUDA;
  }
  return rc == LL_OK ? LL_OK : fail(rc);
}

int ll_set_epilogue(ll_handle h, int epilogue) {
  g_last_error = LL_OK;
  if (!h || epilogue < LL_EPILOGUE_NONE || epilogue > LL_EPILOGUE_GEGLU_TANH) return fail(LL_ERR_INVALID_ARG);
  if (epilogue == LL_EPILOGUE_GEGLU_TANH && h->N % 256 != 0) return fail(LL_ERR_UNSUPPORTED);
  // The GEGLU row order is applied when the weights are copied in.
  if ((epilogue == LL_EPILOGUE_GEGLU_TANH) != is_geglu(h)) h->ready = false;
  h->epilogue = epilogue;
  clear_call_maps(h);  // the width of y may change
  return LL_OK;
}

int ll_set_variant(ll_handle h, int variant) {
  g_last_error = LL_OK;
  if (!h || (variant < LL_VARIANT_AUTO || variant > LL_VARIANT_GEMV))
    return fail(LL_ERR_INVALID_ARG);
  h->variant = variant;
  return LL_OK;
}

int ll_plan(int N, int K, int r, int M, int num_sms, int variant, int* kernel, int* tile_tokens, int* lr_splits) {
  g_last_error = LL_OK;
  if (N < 1 || K < 16 || r < 0 || (N % 8) != 0 || (K % 16) != 0 || M < 1 || num_sms < 2 ||
      (variant < LL_VARIANT_AUTO || variant > LL_VARIANT_GEMV))
    return fail(LL_ERR_INVALID_ARG);
  if (r > 512) return fail(LL_ERR_UNSUPPORTED);
  // A handle-shaped view holding only what the planning reads.
  ll_layer view;
  view.N = N;
  view.K = K;
  view.r = r;
  view.r_pad = (r + 31) / 32 * 32;
  view.klr = (view.r_pad % 64 == 0) ? 64 : 32;
  view.num_sms = num_sms;
  view.variant = variant;
  view.pair_clusters = num_sms / 2;
  const Path path = choose_path(&view, M);
  int kv = LL_VARIANT_SMALL, bt = 128;
  switch (path) {
    case PATH_TC1:
      kv = LL_VARIANT_TC;
      bt = M > 128 ? tc_tile_tokens(&view, M) : 256;
      break;
    case PATH_TC2:
      kv = LL_VARIANT_TC_PAIR;
      bt = tc2_tile_tokens(&view, M);
      break;
    case PATH_STREAM:
      kv = LL_VARIANT_STREAM;
      bt = (M + 15) / 16 * 16;
      break;
    case PATH_F8:
      kv = variant == LL_VARIANT_FP8_ACT ? LL_VARIANT_FP8_ACT : LL_VARIANT_FP8_SPLIT;
      bt = 256;
      break;
    case PATH_F8S:
      kv = variant == LL_VARIANT_FP8_ACT ? LL_VARIANT_FP8_ACT : LL_VARIANT_FP8_SPLIT;
      bt = (M + 15) / 16 * 16;
      break;
    case PATH_GEMV:
      kv = LL_VARIANT_GEMV;
      bt = M;
      break;
    case PATH_SMALL:
      break;
  }
  if (kernel) *kernel = kv;
  if (tile_tokens) *tile_tokens = bt;
  if (lr_splits) *lr_splits = view.r_pad > 0 && path != PATH_GEMV ? plan_lowrank(&view, M).ksplit : 1;
  return LL_OK;
}

int ll_status(ll_handle h) {
  g_last_error = LL_OK;
  if (!h) return fail(LL_ERR_INVALID_ARG);
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  if (v != 0) {
    // A kernel gave up part-way: clear the status and the tile scheduler.
    cudaMemset(h->status, 0, sizeof(int));
    cudaMemset(h->sched, 0, 2 * sizeof(int));
    if (h->f8_cnt) cudaMemset(h->f8_cnt, 0, sizeof(int) * h->f8_cnt_n);
    cudaDeviceSynchronize();
    return LL_ERR_DEVICE_TIMEOUT;
  }
  return LL_OK;
}

int ll_set_debug(ll_handle h, int withhold_producer, uint64_t timeout_ns) {
  g_last_error = LL_OK;
  if (!h || timeout_ns == 0) return fail(LL_ERR_INVALID_ARG);
  h->withhold = withhold_producer ? 1 : 0;
  h->timeout_ns = timeout_ns;
  return LL_OK;
}

int ll_last_launch_count(ll_handle h) { return h ? h->last_launches : 0; }

int ll_set_profiling(ll_handle h, int enable) {
  g_last_error = LL_OK;
  if (!h) return fail(LL_ERR_INVALID_ARG);
  h->profiling = enable ? 1 : 0;
  return LL_OK;
}

int ll_kernel_times(ll_handle h, float* ms, int n) {
  g_last_error = LL_OK;
  if (!h || !h->prof_valid) return -1;
  if (cudaEventSynchronize(h->ev[h->last_launches]) != cudaSuccess) {
    cudaGetLastError();
    fail(LL_ERR_CUDA);
    return -1;
  }
  for (int i = 0; i < h->last_launches && i < n; ++i) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, h->ev[i], h->ev[i + 1]) != cudaSuccess) {
      cudaGetLastError();
      fail(LL_ERR_CUDA);
      return -1;
    }
    if (ms) ms[i] = t;
  }
  return h->last_launches;
}

const char* ll_kernel_name(ll_handle h, int i) {
  if (!h || i < 0 || i >= h->last_launches) return nullptr;
  return h->names[i];
}

int ll_quantize_residual(const void* W, const void* A, const void* B, int N, int K, int r, int scale_mode,
                         void* Q, float* scale, void* stream) {
  g_last_error = LL_OK;
  if (N < 1 || K < 1 || r < 0 || (scale_mode != LL_SCALE_PER_TENSOR && scale_mode != LL_SCALE_PER_ROW))
    return fail(LL_ERR_INVALID_ARG);
  if (!W || !Q || !scale || (r > 0 && (!A || !B))) return fail(LL_ERR_INVALID_ARG);
  if (!aligned(W, 2) || !aligned(scale, 4) || (r > 0 && (!aligned(A, 2) || !aligned(B, 2))))
    return fail(LL_ERR_INVALID_ARG);
  const size_t smem = llk::rq_smem_bytes(K, r);
  if (smem > 227 * 1024) return fail(LL_ERR_UNSUPPORTED);
  if (!is_device_ptr(W) || !is_device_ptr(Q) || !is_device_ptr(scale) ||
      (r > 0 && (!is_device_ptr(A) || !is_device_ptr(B))))
    return fail(LL_ERR_INVALID_ARG);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaFuncSetAttribute(llk::ll_residual_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess ||
      cudaFuncSetAttribute(llk::ll_residual_tensor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int blocks = std::max(1, std::min(N, sms * 4));
  const auto* w = static_cast<const uint16_t*>(W);
  const auto* a = r > 0 ? static_cast<const uint16_t*>(A) : nullptr;
  const auto* b = r > 0 ? static_cast<const uint16_t*>(B) : nullptr;
  auto* q = static_cast<uint8_t*>(Q);
  if (scale_mode == LL_SCALE_PER_ROW) {
    llk::ll_residual_rows_kernel<<<blocks, llk::kRqThreads, smem, st>>>(w, a, b, N, K, r, q, scale, nullptr);
    if (cudaGetLastError() != cudaSuccess) return fail(LL_ERR_CUDA);
    return LL_OK;
  }
  double* rowmax = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&rowmax), sizeof(double) * N, st) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_OOM);
  }
  llk::ll_residual_rows_kernel<<<blocks, llk::kRqThreads, smem, st>>>(w, a, b, N, K, r, q, scale, rowmax);
  llk::ll_residual_tensor_kernel<<<blocks, llk::kRqThreads, smem, st>>>(w, a, b, N, K, r, q, scale, rowmax);
  const bool launched = cudaGetLastError() == cudaSuccess;
  cudaFreeAsync(rowmax, st);
  if (!launched) return fail(LL_ERR_CUDA);
  return LL_OK;
}

int ll_quantize_x(const void* x, int M, int K, int terms, int* e_out, void* hi, void* lo, void* stream) {
  g_last_error = LL_OK;
  if (M < 0 || K < 16 || (K % 16) != 0 || (terms != 1 && terms != 2)) return fail(LL_ERR_INVALID_ARG);
  if (M == 0) return LL_OK;
  if (!x || !e_out || !hi || (terms == 2 && !lo)) return fail(LL_ERR_INVALID_ARG);
  if (!aligned(x, 16) || !aligned(e_out, 4) || !aligned(hi, 16) || (terms == 2 && !aligned(lo, 16)))
    return fail(LL_ERR_INVALID_ARG);
  if (!is_device_ptr(x) || !is_device_ptr(e_out) || !is_device_ptr(hi) || (terms == 2 && !is_device_ptr(lo)))
    return fail(LL_ERR_INVALID_ARG);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  const int blocks = std::max(1, std::min((M + 7) / 8, sms * 8));
  llk::ll_xsplit_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(x), M, K, terms, e_out, static_cast<uint8_t*>(hi), static_cast<uint8_t*>(lo));
  if (cudaGetLastError() != cudaSuccess) return fail(LL_ERR_CUDA);
  return LL_OK;
}

void ll_destroy(ll_handle h) {
  if (!h) return;
  cudaDeviceSynchronize();
  free_layer_mem(h);
  cudaGetLastError();
  delete h;
}

}  // extern "C"

// ===========================================================================
// ll_forward_noalloc: the SMALL kernel chain (down-projection, optional
// split-K reduction, fused residual + low-rank kernel) with every piece of
// scratch in one static device array, for callers that may not allocate.
// Only additions here: the handle-based forward above is untouched.

// File-scope scratch, one instance per GPU on which this module is loaded.
// Host code must not use this name as an address (on the host it is a
// stand-in object); the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LL_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;

struct NoAllocDevice {
  bool ready = false;                // set-up succeeded (a failed set-up is retried by the next call)
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  int num_sms = 0;
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

// Once per device, with that device current: the scratch address, the SM
// count and the kernels' shared-memory limits.  Only a successful set-up
// is kept, so a transient failure does not stick to the device.
NoAllocDevice* noalloc_setup(int dev, int* rc) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) {
    *rc = LL_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    int sms = 0;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0 ||
        cudaFuncSetAttribute(kernel_main(llk::kActNone), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             llk::main_smem_bytes()) != cudaSuccess ||
        cudaFuncSetAttribute(llk::ll_lrdown_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             llk::lr_smem_bytes(256)) != cudaSuccess) {
      cudaGetLastError();
      *rc = LL_ERR_CUDA;
      return nullptr;
    }
    d.scratch = static_cast<unsigned char*>(p);
    d.num_sms = sms;
    d.ready = true;
  }
  *rc = LL_OK;
  return &d;
}

// A per-tensor scale, repeated for each of the N output features.
__global__ void ll_noalloc_scale_kernel(const float* __restrict__ s, float* __restrict__ out, int N) {
  const float v = s[0];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) out[i] = v;
}

size_t round_up256(size_t v) { return (v + 255) / 256 * 256; }

int forward_noalloc(const void* x, const void* A, const void* B, const void* Q, const float* scale, int scale_mode,
                    const void* bias, void* y, int M, int N, int K, int r, cudaStream_t st) {
  using namespace llk;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  int rc = LL_OK;
  NoAllocDevice* d = noalloc_setup(dev, &rc);
  if (!d) return rc;

  // Scratch layout: status word (bytes 0-3; 256 bytes reserved) |
  // broadcast scale (per-tensor only) | t_hi [M, r_pad] | t_lo [M, r_pad].
  const int r_pad = (r + 31) / 32 * 32;
  const size_t t_bytes = static_cast<size_t>(M) * r_pad * sizeof(uint16_t);
  size_t off = 256;
  const size_t scale_off = off;
  if (scale_mode == LL_SCALE_PER_TENSOR) off += round_up256(static_cast<size_t>(N) * sizeof(float));
  const size_t thi_off = off;
  const size_t tlo_off = thi_off + t_bytes;
  if (tlo_off + t_bytes > LL_NOALLOC_SCRATCH_BYTES) return LL_ERR_SCRATCH_LIMIT;

  unsigned char* base = d->scratch;
  int* status = reinterpret_cast<int*>(base);
  const float* scale_n = scale;
  if (scale_mode == LL_SCALE_PER_TENSOR) scale_n = reinterpret_cast<float*>(base + scale_off);
  uint16_t* t_hi = reinterpret_cast<uint16_t*>(base + thi_off);
  uint16_t* t_lo = reinterpret_cast<uint16_t*>(base + tlo_off);

  // Down-projection plan of the SMALL path.
  ll_layer view;
  view.N = N;
  view.K = K;
  view.r = r;
  view.r_pad = r_pad;
  view.num_sms = d->num_sms;
  view.variant = LL_VARIANT_SMALL;
  const LrPlan lp = plan_lowrank(&view, M);

  // Tensor maps over the caller's buffers; rank columns / rows past r read
  // as zeros (TMA fill), which stands in for the zero padding to r_pad.
  CUtensorMap tm_x, tm_q, tm_a, tm_b, tm_thi, tm_tlo, tm_y;
  bool ok = make_map(&tm_x, x, kBF16, M, K, 2ull * K, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&tm_q, Q, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, K, kBK, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= make_map(&tm_y, y, kBF16, M, N, 2ull * N, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (r_pad > 0) {
    ok &= make_map(&tm_a, A, kBF16, N, r, 2ull * r, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&tm_b, B, kBF16, r, K, 2ull * K, kBK, lp.rc, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&tm_thi, t_hi, kBF16, M, r_pad, 2ull * r_pad, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&tm_tlo, t_lo, kBF16, M, r_pad, 2ull * r_pad, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    tm_a = tm_x;  // unused when r_pad == 0
    tm_thi = tm_x;
    tm_tlo = tm_x;
  }
  if (!ok) return LL_ERR_CUDA;

  const Watch watch{status, 2000000000ull};
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  if (scale_mode == LL_SCALE_PER_TENSOR) {
    const int blocks = std::max(1, std::min((N + 255) / 256, 4 * d->num_sms));
    ll_noalloc_scale_kernel<<<blocks, 256, 0, st>>>(scale, const_cast<float*>(scale_n), N);
  }
  if (r_pad > 0) {
    LrDownParams lpp;
    lpp.tm_x = tm_x;
    lpp.tm_b = tm_b;
    lpp.t_hi = t_hi;
    lpp.t_lo = t_lo;
    lpp.M = M;
    lpp.K = K;
    lpp.r_pad = r_pad;
    lpp.rc = lp.rc;
    lpp.tmem_cols = lp.tmem_cols;
    lpp.ksplit = lp.ksplit;
    lpp.kb_per_split = lp.kb_per_split;
    lpp.e_tok = nullptr;
    lpp.wait_prior = 0;
    lpp.watch = watch;
    if (launch_lrdown(lpp, lp, st) != cudaSuccess) {
      cudaGetLastError();
      return LL_ERR_CUDA;
    }
  }
  if (cudaGetLastError() != cudaSuccess) return LL_ERR_CUDA;

  MainParams mp;
  mp.tm_x = tm_x;
  mp.tm_q = tm_q;
  mp.tm_a = tm_a;
  mp.tm_thi = tm_thi;
  mp.tm_tlo = tm_tlo;
  mp.tm_y = tm_y;
  mp.scale = scale_n;
  mp.bias = static_cast<const uint16_t*>(bias);
  mp.M = M;
  mp.N = N;
  mp.K = K;
  mp.r_pad = r_pad;
  mp.n_ftiles = (N + 127) / 128;
  mp.n_ttiles = (M + 127) / 128;
  mp.lr_from_primary = r_pad > 0 ? 1 : 0;
  mp.withhold = 0;
  mp.watch = watch;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = r_pad > 0 ? 1 : 0;
  cfg.gridDim = dim3(std::min(mp.n_ftiles * mp.n_ttiles, d->num_sms));
  cfg.blockDim = dim3(kMainThreads);
  cfg.dynamicSmemBytes = main_smem_bytes();
  if (cudaLaunchKernelEx(&cfg, kernel_main(llk::kActNone), mp) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  return LL_OK;
}

}  // namespace

extern "C" int ll_forward_noalloc(const void* x, const void* A, const void* B, const void* Q, const float* scale,
                                  int scale_mode, const void* bias, void* y, int M, int N, int K, int r,
                                  void* stream) {
  g_last_error = LL_OK;
  if (M < 0 || N < 1 || K < 16 || r < 0 || r > 512 || (N % 8) != 0 || (K % 16) != 0 ||
      (scale_mode != LL_SCALE_PER_TENSOR && scale_mode != LL_SCALE_PER_ROW))
    return fail(LL_ERR_INVALID_ARG);
  if (M == 0) return LL_OK;
  if (r % 8 != 0) return fail(LL_ERR_UNSUPPORTED);
  if (!x || !y || !Q || !scale || (r > 0 && (!A || !B))) return fail(LL_ERR_INVALID_ARG);
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(Q, 16) || !aligned(scale, 4) || (bias && !aligned(bias, 2)) ||
      (r > 0 && (!aligned(A, 16) || !aligned(B, 16))))
    return fail(LL_ERR_INVALID_ARG);
  // y must not overlap any input: the inputs are read in place on every call.
  const size_t ys = static_cast<size_t>(M) * N * 2;
  if (overlaps(y, ys, x, static_cast<size_t>(M) * K * 2) || overlaps(y, ys, Q, static_cast<size_t>(N) * K) ||
      overlaps(y, ys, scale, scale_mode == LL_SCALE_PER_ROW ? 4 * static_cast<size_t>(N) : 4) ||
      (bias && overlaps(y, ys, bias, 2 * static_cast<size_t>(N))) ||
      (r > 0 && (overlaps(y, ys, A, 2 * static_cast<size_t>(N) * r) || overlaps(y, ys, B, 2 * static_cast<size_t>(r) * K))))
    return fail(LL_ERR_INVALID_ARG);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(LL_ERR_CUDA);
  }
  if (!is_device_ptr_on(x, dev) || !is_device_ptr_on(y, dev) || !is_device_ptr_on(Q, dev) ||
      !is_device_ptr_on(scale, dev) || (bias && !is_device_ptr_on(bias, dev)) ||
      (r > 0 && (!is_device_ptr_on(A, dev) || !is_device_ptr_on(B, dev))))
    return fail(LL_ERR_INVALID_ARG);
  const int rc = forward_noalloc(x, A, B, Q, scale, scale_mode, bias, y, M, N, K, r, static_cast<cudaStream_t>(stream));
  return rc == LL_OK ? LL_OK : fail(rc);
}
