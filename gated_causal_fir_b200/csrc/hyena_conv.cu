// hyena_conv.cu -- host side of the C ABI declared in include/hyena_conv.h: argument checks,
// algorithm selection, TMA descriptor encoding and kernel launches.  Every step of the
// computation runs in the kernels of fir_tc.cuh and fir_cuda_core.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <limits>
#include <mutex>
#include <type_traits>

#include "hyena_conv.h"
#include "hyena_conv_testing.h"
#include "fir_bwd.cuh"
#include "fir_cuda_core.cuh"
#include "fir_fft.cuh"
#include "fir_fftblk.cuh"
#include "fir_tc.cuh"
#include "fir_tc_bwd.cuh"

namespace {

using hyena::cc::WindowParams;

#ifndef HYENA_TC_L2_PROMOTION
#define HYENA_TC_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_NONE
#endif
#ifndef HYENA_TC_PAIRED
#define HYENA_TC_PAIRED 1
#endif
#ifndef HYENA_PDL
#define HYENA_PDL 1
#endif


constexpr int kMaxDevices = 64;
// Shared memory of the dh partial kernel at 64 channels per piece: dz rows + x window.
constexpr int kDhSmemMax =
    ((2 * hyena::bwd::kDhRows + hyena::bwd::kDhTaps - 1) * (64 + 1) + hyena::bwd::kDhRedFloats) *
    static_cast<int>(sizeof(float));
constexpr int kMaxWindowTaps = 16;
constexpr int kBlkThreads = 512;  // block FFT: one CTA of 512 threads per SM
#ifndef HYENA_WINDOW_ROWS
#define HYENA_WINDOW_ROWS 128
#endif
constexpr int kWindowRows = HYENA_WINDOW_ROWS;

struct DeviceState {
  std::once_flag once;
  int sm_count = 0;
  cudaError_t err = cudaSuccess;
};
DeviceState g_devices[kMaxDevices];

// Per-device one-time set-up: SM count and the tensor-core kernel's shared-memory opt-in.
int current_device(DeviceState *&ds) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HYENA_ERR_CUDA;
  ds = &g_devices[dev];
  DeviceState *d = ds;
  std::call_once(d->once, [d, dev]() {
    cudaError_t e = cudaDeviceGetAttribute(&d->sm_count, cudaDevAttrMultiProcessorCount, dev);
    // Every (groups per tile, history tiles) instantiation with its shared-memory size.
    const struct {
      const void *fn;
      int smem;
    } kernels[] = {
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 1>), hyena::tc::Layout<1>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 2>), hyena::tc::Layout<2>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 3>), hyena::tc::Layout<3>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 4>), hyena::tc::Layout<4>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 5>), hyena::tc::Layout<5>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<2, 1>), hyena::tc::Layout<1>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<2, 2>), hyena::tc::Layout<2>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<4, 1>), hyena::tc::Layout<1>::kSmemBytes},
        {reinterpret_cast<const void *>(hyena::tc::fir_tc_kernel<1, 1, true>), hyena::tc::Layout<1>::kSmemBytes}};
    for (const auto &k : kernels)
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
    const void *dh_kernels[] = {
        reinterpret_cast<const void *>(hyena::bwd::fir_bwd_dh_partial_kernel<float>),
        reinterpret_cast<const void *>(hyena::bwd::fir_bwd_dh_partial_kernel<__nv_bfloat16>)};
    for (const void *k : dh_kernels)
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kDhSmemMax);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void *>(hyena::tcb::fir_tc_bwd_kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               hyena::tcb::kSmemBytes);
    // block FFT instantiations (see kBlkConfigs)
    const struct {
      const void *fn;
      int smem;
    } blk[] = {
#define HYENA_BLK_ATTR(T, LGN, PP, SQ)                                                          \
  {reinterpret_cast<const void *>(hyena::fftblk::fir_fftblk_kernel<T, LGN, PP, kBlkThreads, SQ>), \
   hyena::fftblk::Smem<T, LGN, PP, SQ>::kBytes}
        HYENA_BLK_ATTR(__nv_bfloat16, 10, 8, true), HYENA_BLK_ATTR(__nv_bfloat16, 11, 4, true),
        HYENA_BLK_ATTR(__nv_bfloat16, 12, 2, true), HYENA_BLK_ATTR(__nv_bfloat16, 13, 1, false),
        HYENA_BLK_ATTR(float, 10, 4, true), HYENA_BLK_ATTR(float, 11, 2, true),
        HYENA_BLK_ATTR(float, 12, 1, true)
#undef HYENA_BLK_ATTR
    };
    for (const auto &k : blk)
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
    const void *tiled[] = {
        reinterpret_cast<const void *>(hyena::cc::fir_tiled_kernel<float, false>),
        reinterpret_cast<const void *>(hyena::cc::fir_tiled_kernel<float, true>),
        reinterpret_cast<const void *>(hyena::cc::fir_tiled_kernel<__nv_bfloat16, false>),
        reinterpret_cast<const void *>(hyena::cc::fir_tiled_kernel<__nv_bfloat16, true>)};
    for (const void *k : tiled)
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 hyena::cc::kTileSmemBytes);

    d->err = e;
  });
  return d->err == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct Problem {
  const void *q, *k, *v;
  const float *h;
  void *y;
  int64_t B, L, D;
  int d_g, l_h, l_b, dtype;
  const void *kh = nullptr, *vh = nullptr;  // [B, Lh, D] rows before row 0 (Lh = 0: zeros)
  int64_t Lh = 0;
  int64_t elem() const { return dtype == HYENA_DTYPE_F32 ? 4 : 2; }
  int64_t numel() const { return B * L * D; }
  int64_t G() const { return D / d_g; }
};

constexpr int kEmpty = -1;  // internal: valid problem with nothing to compute

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, const void *b, int64_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + static_cast<uintptr_t>(bytes) && y < x + static_cast<uintptr_t>(bytes);
}

// Host-side checks shared by every forward entry point (no device access).
int validate(const Problem &P) {
  if (P.dtype != HYENA_DTYPE_BF16 && P.dtype != HYENA_DTYPE_F32) return HYENA_ERR_INVALID_ARG;
  if (P.B < 0 || P.L < 0 || P.D < 1 || P.d_g < 1 || P.l_h < 1 || P.l_b < 1)
    return HYENA_ERR_INVALID_ARG;
  if (P.D % P.d_g != 0) return HYENA_ERR_INVALID_ARG;
  if (P.B == 0 || P.L == 0) return kEmpty;
  const int64_t lim = std::numeric_limits<int64_t>::max() / 8;
  if (P.B > lim / P.L || P.B * P.L > lim / P.D) return HYENA_ERR_INVALID_ARG;
  if (!P.q || !P.k || !P.v || !P.h || !P.y) return HYENA_ERR_INVALID_ARG;
  const uintptr_t es = static_cast<uintptr_t>(P.elem());
  if (!aligned(P.q, es) || !aligned(P.k, es) || !aligned(P.v, es) || !aligned(P.y, es) ||
      !aligned(P.h, 4))
    return HYENA_ERR_MISALIGNED;
  const int64_t bytes = P.numel() * P.elem();
  if (overlaps(P.y, P.q, bytes) || overlaps(P.y, P.k, bytes) || overlaps(P.y, P.v, bytes))
    return HYENA_ERR_INVALID_ARG;
  if (P.Lh > 0) {
    if (!P.kh || !P.vh || P.Lh > lim / P.B / P.D) return HYENA_ERR_INVALID_ARG;
    if (!aligned(P.kh, es) || !aligned(P.vh, es)) return HYENA_ERR_MISALIGNED;
    const int64_t hb = P.B * P.Lh * P.D * P.elem();
    // y must not overlap the history either (the intervals differ in length)
    const uintptr_t y0 = reinterpret_cast<uintptr_t>(P.y);
    for (const void *hp : {P.kh, P.vh}) {
      const uintptr_t h0 = reinterpret_cast<uintptr_t>(hp);
      if (y0 < h0 + static_cast<uintptr_t>(hb) && h0 < y0 + static_cast<uintptr_t>(bytes))
        return HYENA_ERR_INVALID_ARG;
    }
  }
  return HYENA_OK;
}

bool all_aligned16(const Problem &P) {
  return aligned(P.q, 16) && aligned(P.k, 16) && aligned(P.v, 16) && aligned(P.y, 16) &&
         (P.Lh == 0 || (aligned(P.kh, 16) && aligned(P.vh, 16)));
}

// Tensor-core plan: history rows, history tiles, one group's band width in TMEM columns and the
// number of band sets (2 when they fit, else 1; 0 = does not fit).
struct TcPlan {
  int halo, nh, band_cols, ng, nbuf;
};

TcPlan tc_plan(const Problem &P) {
  TcPlan t{0, 0, 0, 0, 0};
  if (P.d_g != 16 && P.d_g != 32 && P.d_g != 64) return t;
  if (P.l_h - 1 > hyena::tc::kMaxHalo) return t;
  t.halo = ((P.l_h - 1) + 15) / 16 * 16;
  t.nh = t.halo <= hyena::tc::kTM ? 1 : (t.halo + hyena::tc::kTM - 1) / hyena::tc::kTM;
  t.band_cols = (hyena::tc::kTM + t.halo) / 2;
  t.ng = hyena::tc::kNC / P.d_g;
  const int room = hyena::tc::kTmemCols - hyena::tc::kBandCol0;
  t.nbuf = 2 * t.ng * t.band_cols <= room ? 2 : (t.ng * t.band_cols <= room ? 1 : 0);
  return t;
}

bool tensor_supported(const Problem &P) {
  const int64_t i32 = std::numeric_limits<int32_t>::max();
  return P.dtype == HYENA_DTYPE_BF16 && P.D % hyena::tc::kNC == 0 && tc_plan(P).nbuf > 0 &&
         all_aligned16(P) && P.L <= i32 && P.B <= i32 && P.D <= i32 && P.Lh <= i32;
}

bool window_supported(const Problem &P) {
  const int vec = P.dtype == HYENA_DTYPE_F32 ? 4 : 8;
  return P.l_h <= kMaxWindowTaps && P.d_g % vec == 0 && all_aligned16(P);
}

// Block FFT (overlap-save, fir_fftblk_kernel): transform length N = 2^lgn with P channel pairs
// per CTA (P N = 8192 complex values in shared memory for bf16, 4096 for fp32, whose staged
// rows are twice as wide), M = N - l_h + 1 outputs per block; one CTA per SM.
struct BlkConfig {
  int lgn, P;
};
constexpr BlkConfig kBlkBf16[] = {{10, 8}, {11, 4}, {12, 2}, {13, 1}};
constexpr BlkConfig kBlkF32[] = {{10, 4}, {11, 2}, {12, 1}};

// Time per point of each transform length relative to N = 1024 and 2048 (see blk_plan).
double blk_weight(int lgn) { return lgn <= 11 ? 1.0 : (lgn == 12 ? 2.2 : 2.6); }

struct BlkPlan {
  BlkConfig cfg;
  int M, nTB;
  bool ok;
};

// The transform length with the least estimated time: N log N per block times the blocks per
// sequence, weighted by how fast each length's kernel runs per point (measured on the MR shape:
// ~80 ns per 8192 complex points at N = 1024 and 2048, ~2.2x that at N = 4096 and ~2.6x at
// 8192, whose narrower row pieces of 2 and 1 channel pairs per CTA make the staging copies
// small), among the lengths whose channel block (2P channels) lies inside one group, whose row
// vectors are aligned and whose blocks keep at least N / 8 rows (or one block covers the
// sequence); ok = false when none applies.
BlkPlan blk_plan(const Problem &P) {
  BlkPlan best{kBlkBf16[0], 0, 0, false};
  double best_cost = 0;
  const bool f32 = P.dtype == HYENA_DTYPE_F32;
  const int ncfg = f32 ? 3 : 4;
  for (int ci = 0; ci < ncfg; ++ci) {
    const BlkConfig &c = f32 ? kBlkF32[ci] : kBlkBf16[ci];
    const int64_t N = int64_t{1} << c.lgn;
    if (N < P.l_h || P.d_g % (2 * c.P) != 0 || P.D % (2 * c.P) != 0) continue;
    const uintptr_t vec = std::min<uintptr_t>(16, static_cast<uintptr_t>(2 * c.P * P.elem()));
    if (!aligned(P.q, vec) || !aligned(P.k, vec) || !aligned(P.v, vec) || !aligned(P.y, vec) ||
        (P.Lh > 0 && (!aligned(P.kh, vec) || !aligned(P.vh, vec))))
      continue;
    const int64_t M = N - P.l_h + 1, nTB = (P.L + M - 1) / M;
    // blocks that keep less than an eighth of their rows cost more than the direct sum
    if (M < N / 8 && nTB > 1) continue;
    if (P.D / (2 * c.P) * nTB > std::numeric_limits<int32_t>::max()) continue;
    const double cost = static_cast<double>(nTB) * static_cast<double>(N) * c.lgn * blk_weight(c.lgn);
    if (!best.ok || cost < best_cost) {
      best = BlkPlan{c, static_cast<int>(M), static_cast<int>(nTB), true};
      best_cost = cost;
    }
  }
  return best;
}

bool fftblk_supported(const Problem &P) { return blk_plan(P).ok; }

// AUTO's choice between the block FFT and the direct sum: flops per output channel, ~5 N log2 N
// per length-N transform (forward and inverse, two channels per transform) against 2 l_h, the
// FFT's weighted by how much faster per flop its kernel runs.
#ifndef HYENA_FFT_FLOP_WEIGHT
#define HYENA_FFT_FLOP_WEIGHT 0.5
#endif
bool fftblk_beats_direct(const Problem &P) {
  const BlkPlan bp = blk_plan(P);
  if (!bp.ok) return false;
  const double fft = HYENA_FFT_FLOP_WEIGHT * blk_weight(bp.cfg.lgn) * 5.0 * bp.nTB *
                     static_cast<double>(1 << bp.cfg.lgn) * bp.cfg.lgn / static_cast<double>(P.L);
  return fft < 2.0 * P.l_h;
}

// MMAs one 128-row tile issues on the tensor path (groups per tile x k-steps).  Each costs
// ~55 cycles of issue at any N <= 64; past ~24 per tile the issuing thread, not HBM, sets the
// pace, and for short filters the CUDA-core window kernel is faster (measured on the SE
// workload: 36 MMAs per tile, 80 us on tensor cores vs 50 us in the window kernel).
constexpr int kMaxTileMmas = 24;

#ifndef HYENA_FFT_MIN_TAPS
#define HYENA_FFT_MIN_TAPS 17
#endif

int select_algo(const Problem &P) {
  const bool tensor = tensor_supported(P), window = window_supported(P);
  const bool fft = P.l_h >= HYENA_FFT_MIN_TAPS && fftblk_beats_direct(P);
  if (tensor && window) {
    const TcPlan t = tc_plan(P);
    return t.ng * ((hyena::tc::kTM + t.halo) / 16) <= kMaxTileMmas ? HYENA_ALGO_TENSOR
                                                                   : HYENA_ALGO_WINDOW;
  }
  if (tensor) return HYENA_ALGO_TENSOR;  // up to 641 taps it beats the block FFT (50-108 us
                                         // against 170-250 us at the MR shape)
  if (window) return HYENA_ALGO_WINDOW;
  if (fft) return HYENA_ALGO_FFT;
  return HYENA_ALGO_DIRECT;
}

// Test hooks of the tensor-core forward (hyena_testing_fwd_fault): a shorter limit for the
// waits between roles, and an arrive the MMA issuer withholds.  Zero = the product behaviour.
struct TcTestHooks {
  unsigned long long wait_ns = 0;
  int fault = 0;
};

int launch_tensor(const Problem &P, cudaStream_t s, const TcTestHooks &hooks = TcTestHooks()) {
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return HYENA_ERR_CUDA;
  // q, k, v, y over [B, L, D]; then k, v history over [B, Lh, D] (without history the k, v
  // maps stand in: the kernel never reads them then).
  CUtensorMap maps[6];
  const bool hist = P.Lh > 0;
  const void *ptrs[6] = {P.q, P.k, P.v, P.y, hist ? P.kh : P.k, hist ? P.vh : P.v};
  const cuuint32_t box[3] = {hyena::tc::kNC, hyena::tc::kTM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  for (int i = 0; i < 6; ++i) {
    const cuuint64_t rows = static_cast<cuuint64_t>(i >= 4 && hist ? P.Lh : P.L);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(P.D), rows, static_cast<cuuint64_t>(P.B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(P.D) * 2,
                                   rows * static_cast<cuuint64_t>(P.D) * 2};
    if (enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptrs[i]), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            HYENA_TC_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return HYENA_ERR_CUDA;
  }
  const TcPlan plan = tc_plan(P);
  hyena::tc::Params p;
  p.h = P.h;
  p.q = static_cast<const __nv_bfloat16 *>(P.q);
  p.y = static_cast<__nv_bfloat16 *>(P.y);
  p.k = static_cast<const __nv_bfloat16 *>(P.k);
  p.v = static_cast<const __nv_bfloat16 *>(P.v);
  p.kh = static_cast<const __nv_bfloat16 *>(hist ? P.kh : P.k);
  p.vh = static_cast<const __nv_bfloat16 *>(hist ? P.vh : P.v);
  p.D = P.D;
  p.wait_ns = hooks.wait_ns ? hooks.wait_ns : hyena::kWaitTimeoutNs;
  p.fault = hooks.fault;
  p.B = static_cast<int>(P.B);
  p.L = static_cast<int>(P.L);
  p.CB = static_cast<int>(P.D / hyena::tc::kNC);
  p.l_h = P.l_h;
  p.halo = plan.halo;
  p.band_cols = plan.band_cols;
  p.nbuf = plan.nbuf;
  p.nT = static_cast<int>((P.L + hyena::tc::kTM - 1) / hyena::tc::kTM);
  p.hist_tiles = hist ? plan.nh : 0;
  p.Lh = static_cast<int>(P.Lh);
  const long long sms = ds->sm_count;
  p.paired = HYENA_TC_PAIRED && p.CB % 2 == 0 && sms >= 2;
  long long grid;
  if (p.paired) {
    p.W = static_cast<long long>(p.CB / 2) * p.B * p.nT;
    grid = 2 * (p.W < sms / 2 ? p.W : sms / 2);
  } else {
    p.W = static_cast<long long>(p.CB) * p.B * p.nT;
    grid = p.W < sms ? p.W : sms;
  }
  const unsigned g = static_cast<unsigned>(grid);
  constexpr int T = hyena::tc::kThreads;
  // Programmatic dependent launch: the kernel's set-up (barriers, tensor memory) overlaps the
  // tail of the previous kernel in the stream; it reads nothing before that kernel is done.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = HYENA_PDL;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(g);
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = 0;  // set per instantiation below
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
#define HYENA_TC_LAUNCH(NG, NH)                                                            \
  cfg.dynamicSmemBytes = hyena::tc::Layout<NH>::kSmemBytes;                                  \
  le = cudaLaunchKernelEx(&cfg, hyena::tc::fir_tc_kernel<NG, NH>, maps[0], maps[1], maps[2], \
                          maps[3], maps[4], maps[5], p)
  if (hooks.wait_ns || hooks.fault) {  // the test instantiation (one group, one history tile)
    if (plan.ng != 1 || plan.nh != 1) return HYENA_ERR_UNSUPPORTED;
    cfg.dynamicSmemBytes = hyena::tc::Layout<1>::kSmemBytes;
    le = cudaLaunchKernelEx(&cfg, hyena::tc::fir_tc_kernel<1, 1, true>, maps[0], maps[1], maps[2],
                            maps[3], maps[4], maps[5], p);
    return le == cudaSuccess && cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
  }
  switch (plan.ng * 8 + plan.nh) {
    case 9: HYENA_TC_LAUNCH(1, 1); break;
    case 10: HYENA_TC_LAUNCH(1, 2); break;
    case 11: HYENA_TC_LAUNCH(1, 3); break;
    case 12: HYENA_TC_LAUNCH(1, 4); break;
    case 13: HYENA_TC_LAUNCH(1, 5); break;
    case 17: HYENA_TC_LAUNCH(2, 1); break;
    case 18: HYENA_TC_LAUNCH(2, 2); break;
    case 33: HYENA_TC_LAUNCH(4, 1); break;
    default: return HYENA_ERR_UNSUPPORTED;
  }
#undef HYENA_TC_LAUNCH
  return le == cudaSuccess && cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

// Time steps per thread of the window kernel: as many as make the whole problem one full wave
// of resident threads (SMs x resident blocks x block), so that every SM gets the same number of
// rows, within [kWindowMinRows, kWindowRows] (a longer run where even kWindowRows per thread
// needs more than one wave).
#ifndef HYENA_WINDOW_WAVE
#define HYENA_WINDOW_WAVE 1
#endif
constexpr int kWindowMinRows = 32;  // halo (l_h - 1 rows) at most ~half a run at l_h = 16

// Resident blocks per SM of `kernel` at `block` threads on the current device, queried once per
// (kernel, device) through the caller's cache.
template <typename K>
int resident_blocks(K kernel, int block, std::atomic<int> (&cache)[kMaxDevices], int &per_sm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HYENA_ERR_CUDA;
  per_sm = cache[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block, 0) != cudaSuccess)
      return HYENA_ERR_CUDA;
    per_sm = per_sm > 0 ? per_sm : 1;
    cache[dev].store(per_sm, std::memory_order_relaxed);
  }
  return HYENA_OK;
}

// A kernel launch, with programmatic stream serialisation where `pdl` (the kernel then waits
// for the previous kernels of the stream itself, with griddepcontrol.wait).
template <typename... Exp, typename... Act>
cudaError_t launch_ex(bool pdl, void (*kernel)(Exp...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, Act &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl && HYENA_PDL;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Act>(args)...);
}

// Run length of the window kernels: with `units` thread columns per time block and `wave`
// resident threads, the rows that make the whole problem one full wave.
long long window_rows(long long units, long long L, long long wave) {
  long long rows = kWindowRows;
  const long long tb_per_wave = wave / units;  // time blocks one wave holds
  if (HYENA_WINDOW_WAVE && tb_per_wave >= 1 && units * ((L + kWindowRows - 1) / kWindowRows) <= wave) {
    rows = (L + tb_per_wave - 1) / tb_per_wave;  // ceil(L / rows) <= tb_per_wave
    rows = std::max<long long>(rows, kWindowMinRows);
    rows = std::min<long long>(rows, kWindowRows);
  }
  return rows;
}

template <typename T, int LH>
int launch_window_lh(const Problem &P, WindowParams wp, int sm_count, cudaStream_t s) {
  const auto kernel = hyena::cc::fir_window_kernel<T, LH>;
  static std::atomic<int> resident[kMaxDevices];  // blocks per SM per device (0: not queried)
  int per_sm = 0;
  if (resident_blocks(kernel, hyena::cc::kWindowBlock, resident, per_sm) != HYENA_OK)
    return HYENA_ERR_CUDA;
  const long long wave = static_cast<long long>(sm_count) * per_sm * hyena::cc::kWindowBlock;
  const long long units = wp.B * wp.cv;  // thread columns per time block
  const long long rows = window_rows(units, wp.L, wave);
  wp.rows = static_cast<int>(rows);
  wp.n_tb = (wp.L + rows - 1) / rows;
  const long long threads = units * wp.n_tb;
  const long long blocks = (threads + hyena::cc::kWindowBlock - 1) / hyena::cc::kWindowBlock;
  if (blocks > std::numeric_limits<int32_t>::max()) return HYENA_ERR_UNSUPPORTED;
  if (launch_ex(true, kernel, dim3(static_cast<unsigned>(blocks)), dim3(hyena::cc::kWindowBlock), 0,
                s, static_cast<const T *>(P.q), static_cast<const T *>(P.k),
                static_cast<const T *>(P.v), static_cast<const float *>(P.h),
                static_cast<T *>(P.y), wp) != cudaSuccess)
    return HYENA_ERR_CUDA;
  return HYENA_OK;
}

template <typename T, int LH = 1>
int launch_window_dispatch(const Problem &P, const WindowParams &wp, int sm_count,
                           cudaStream_t s) {
  if constexpr (LH <= kMaxWindowTaps) {
    if (P.l_h == LH) return launch_window_lh<T, LH>(P, wp, sm_count, s);
    return launch_window_dispatch<T, LH + 1>(P, wp, sm_count, s);
  }
  return HYENA_ERR_UNSUPPORTED;
}

int launch_window(const Problem &P, cudaStream_t s) {
  const int vec = P.dtype == HYENA_DTYPE_F32 ? 4 : 8;
  WindowParams wp;
  wp.B = P.B;
  wp.L = P.L;
  wp.D = P.D;
  wp.d_g = P.d_g;
  wp.cv = P.D / vec;
  wp.kh = P.kh;
  wp.vh = P.vh;
  wp.Lh = P.Lh;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  const int rc = P.dtype == HYENA_DTYPE_F32
                     ? launch_window_dispatch<float>(P, wp, ds->sm_count, s)
                     : launch_window_dispatch<__nv_bfloat16>(P, wp, ds->sm_count, s);
  if (rc != HYENA_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

// The tiled direct sum (fir_tiled_kernel): forward (y) or, with kAnti, the backward's
// transposed product (dk, dv from q, dy).  Persistent CTAs over the tiles.
// run_if (anti only): the kernel's gate word, run_token the value that lets it run; a gated
// launch takes one block per SM and starts early (programmatic dependent launch), so that it
// costs little when the word does not match.
template <typename T, bool kAnti>
int launch_tiled(const Problem &P, const void *dy, void *out0, void *out1, cudaStream_t s,
                 const unsigned *run_if = nullptr, unsigned run_token = 0) {
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  namespace cc = hyena::cc;
  const long long tiles = P.B * ((P.L + cc::kTileR - 1) / cc::kTileR) *
                          ((P.D + cc::kTileC - 1) / cc::kTileC);
  const long long grid =
      std::min<long long>(tiles, static_cast<long long>(ds->sm_count) * (run_if ? 1 : 4));
  const cudaError_t e = launch_ex(
      run_if != nullptr, cc::fir_tiled_kernel<T, kAnti>, dim3(static_cast<unsigned>(grid)),
      dim3(cc::kTileThreads), cc::kTileSmemBytes, s, static_cast<const T *>(P.q),
      static_cast<const T *>(dy), static_cast<const T *>(P.k), static_cast<const T *>(P.v), P.h,
      static_cast<T *>(out0), static_cast<T *>(out1), P.B, P.L, P.D, P.d_g, P.l_h,
      static_cast<const T *>(P.kh), static_cast<const T *>(P.vh), P.Lh, run_if, run_token);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

template <typename T, int LGN, int PP, bool SQ>
int launch_fftblk_cfg(const Problem &P, const BlkPlan &bp, int sm_count, cudaStream_t s) {
  hyena::fftblk::BlkParams p;
  p.q = P.q;
  p.k = P.k;
  p.v = P.v;
  p.kh = P.Lh > 0 ? P.kh : P.k;
  p.vh = P.Lh > 0 ? P.vh : P.v;
  p.h = P.h;
  p.y = P.y;
  p.L = P.L;
  p.D = P.D;
  p.Lh = P.Lh;
  p.CB = static_cast<int>(P.D / (2 * PP));
  p.nTB = bp.nTB;
  p.M = bp.M;
  p.d_g = P.d_g;
  p.l_h = P.l_h;
  // siblings: enough consecutive channel blocks for 64 bytes of a row (one DRAM access)
  p.Q = std::max(1, 64 / static_cast<int>(2 * PP * P.elem()));
  while (p.CB % p.Q != 0) p.Q /= 2;
  p.items = P.B * (p.CB / p.Q) * static_cast<long long>(p.nTB);
  const long long groups = std::max<long long>(1, static_cast<long long>(sm_count) / p.Q);
  const long long grid = std::min<long long>(p.items, groups) * p.Q;
  if (launch_ex(true, hyena::fftblk::fir_fftblk_kernel<T, LGN, PP, kBlkThreads, SQ>,
                dim3(static_cast<unsigned>(grid)), dim3(kBlkThreads),
                hyena::fftblk::Smem<T, LGN, PP, SQ>::kBytes, s, p) != cudaSuccess)
    return HYENA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

int launch_fftblk(const Problem &P, cudaStream_t s) {
  const BlkPlan bp = blk_plan(P);
  if (!bp.ok) return HYENA_ERR_UNSUPPORTED;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  const int sms = ds->sm_count;
  if (P.dtype == HYENA_DTYPE_F32) {
    switch (bp.cfg.lgn) {
      case 10: return launch_fftblk_cfg<float, 10, 4, true>(P, bp, sms, s);
      case 11: return launch_fftblk_cfg<float, 11, 2, true>(P, bp, sms, s);
      case 12: return launch_fftblk_cfg<float, 12, 1, true>(P, bp, sms, s);
      default: return HYENA_ERR_UNSUPPORTED;
    }
  }
  switch (bp.cfg.lgn) {
    case 10: return launch_fftblk_cfg<__nv_bfloat16, 10, 8, true>(P, bp, sms, s);
    case 11: return launch_fftblk_cfg<__nv_bfloat16, 11, 4, true>(P, bp, sms, s);
    case 12: return launch_fftblk_cfg<__nv_bfloat16, 12, 2, true>(P, bp, sms, s);
    case 13: return launch_fftblk_cfg<__nv_bfloat16, 13, 1, false>(P, bp, sms, s);
    default: return HYENA_ERR_UNSUPPORTED;
  }
}

int launch_direct(const Problem &P, cudaStream_t s) {
  if (P.dtype == HYENA_DTYPE_F32) return launch_tiled<float, false>(P, nullptr, P.y, nullptr, s);
  return launch_tiled<__nv_bfloat16, false>(P, nullptr, P.y, nullptr, s);
}

int run(const Problem &P, int algo, cudaStream_t s) {
  const int rc = validate(P);
  if (rc == kEmpty) return HYENA_OK;
  if (rc != HYENA_OK) return rc;
  switch (algo) {
    case HYENA_ALGO_AUTO:
      algo = select_algo(P);
      break;
    case HYENA_ALGO_TENSOR:
      if (!tensor_supported(P)) return HYENA_ERR_UNSUPPORTED;
      break;
    case HYENA_ALGO_WINDOW:
      if (!window_supported(P)) return HYENA_ERR_UNSUPPORTED;
      break;
    case HYENA_ALGO_FFT:
      if (!fftblk_supported(P)) return HYENA_ERR_UNSUPPORTED;
      break;
    case HYENA_ALGO_DIRECT:
      break;
    default:
      return HYENA_ERR_INVALID_ARG;
  }
  if (algo == HYENA_ALGO_TENSOR) return launch_tensor(P, s);
  if (algo == HYENA_ALGO_WINDOW) return launch_window(P, s);
  if (algo == HYENA_ALGO_FFT) return launch_fftblk(P, s);
  return launch_direct(P, s);
}

// ------------------------------------------------------------------------------ backward
struct BwdPlan {
  int cp, npieces, nchunk;
  int64_t partial_floats;
};

BwdPlan bwd_plan(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  BwdPlan b;
  b.cp = hyena::bwd::dh_piece(d_g);
  b.npieces = static_cast<int>(D / b.cp);
  b.nchunk = static_cast<int>((L + hyena::bwd::kDhRows - 1) / hyena::bwd::kDhRows);
  b.partial_floats = B * b.nchunk * static_cast<int64_t>(b.npieces) * l_h;
  return b;
}

int64_t round256(int64_t n) { return (n + 255) / 256 * 256; }

// Workspace of the tensor-core backward: one dh partial (l_h floats) and one group id per
// (CTA, segment) slot, then one segment count per CTA.
constexpr int64_t kTcBwdMaxGrid = 1024;
struct TcBwdLayout {
  int64_t off_group, off_count, bytes;
};
TcBwdLayout tc_bwd_layout(int64_t slots, int64_t grid, int l_h) {
  TcBwdLayout o;
  o.off_group = round256(slots * l_h * 4);
  o.off_count = o.off_group + round256(slots * 4);
  o.bytes = o.off_count + round256(grid * 4);
  return o;
}

// Upper bound over every grid size: a CTA of a walk of W tiles split over `grid` CTAs touches
// at most per / nT + 2 sequences, so slots <= B G + 2 grid.
int64_t tc_bwd_bytes_bound(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  if (d_g != hyena::tc::kNC || D % hyena::tc::kNC != 0) return 0;
  const int64_t nT = (L + hyena::tc::kTM - 1) / hyena::tc::kTM, G = D / hyena::tc::kNC;
  const int64_t W = G * B * nT;
  const int64_t grid = W < kTcBwdMaxGrid ? W : kTcBwdMaxGrid;
  return tc_bwd_layout(B * G + 2 * grid, grid, l_h).bytes;
}

// Partials of fir_bwd_window_kernel for any dtype: one per thread (4 channels at fp32) and time
// block.  With `min_rows`-row time blocks (the shortest run the launch picks) every run length
// fits; with one time block the launch lengthens the runs to fit whatever it is given.
int64_t window_bwd_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h, int64_t min_rows) {
  if (l_h > kMaxWindowTaps || d_g % 4 != 0) return 0;
  return round256(B * ((L + min_rows - 1) / min_rows) * (D / 4) * l_h * 4);
}

// The workspace a backward call needs at least (every algorithm runs in it) ...
// The partials of every algorithm fit below this offset; the tensor-core path keeps its
// operand-range flag at it (the fp32 fallback behind that path reuses the partials' room).
int64_t bwd_flag_offset(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  const int64_t cc = round256(bwd_plan(B, L, D, d_g, l_h).partial_floats * 4);
  const int64_t tc = tc_bwd_bytes_bound(B, L, D, d_g, l_h);
  const int64_t win = window_bwd_bytes(B, L, D, d_g, l_h, std::max<int64_t>(L, 1));
  return std::max(cc, std::max(tc, win));
}

int64_t bwd_required_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  if (B == 0 || L == 0) return 0;  // nothing runs but the zeroing of dh
  return bwd_flag_offset(B, L, D, d_g, l_h) + 256;
}

// ... and the size hyena_conv_bwd_workspace_bytes reports: enough for the window kernel's
// shortest runs as well.
int64_t bwd_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  return std::max(bwd_required_bytes(B, L, D, d_g, l_h),
                  window_bwd_bytes(B, L, D, d_g, l_h, kWindowMinRows));
}

// The CUDA-core kernels' index limits: one 32-bit grid of (chunk, piece, sequence) blocks, and
// the reduction's terms per group.
bool cuda_core_bwd_launchable(const Problem &P) {
  const BwdPlan b = bwd_plan(P.B, P.L, P.D, P.d_g, P.l_h);
  const int64_t i32 = std::numeric_limits<int32_t>::max();
  return b.nchunk <= i32 && P.B <= i32 && P.B * b.nchunk * static_cast<int64_t>(b.npieces) <= i32 &&
         P.B * b.nchunk * (P.d_g / b.cp) <= i32;
}

// run_if, run_token: as fir_tiled_kernel's (null: always run).
template <typename T>
int launch_bwd_cuda_core(const Problem &P, const void *dy, void *dk, void *dv, float *dh,
                         float *partial, cudaStream_t s, const unsigned *run_if = nullptr,
                         unsigned run_token = 0) {
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  const long long cap = static_cast<long long>(ds->sm_count) * 16;
  const int rt = launch_tiled<T, true>(P, dy, dk, dv, s, run_if, run_token);  // dk, dv
  if (rt != HYENA_OK) return rt;
  if (!cuda_core_bwd_launchable(P)) return HYENA_ERR_UNSUPPORTED;
  const BwdPlan b = bwd_plan(P.B, P.L, P.D, P.d_g, P.l_h);
  // gated: one block per SM walks every (chunk, piece, sequence); else one block each
  const long long nblk = P.B * b.nchunk * static_cast<long long>(b.npieces);
  const long long grid = run_if ? std::min<long long>(nblk, ds->sm_count) : nblk;
  const int smem = ((2 * hyena::bwd::kDhRows + hyena::bwd::kDhTaps - 1) * (b.cp + 1) +
                    hyena::bwd::kDhRedFloats) * 4;
  if (launch_ex(run_if != nullptr, hyena::bwd::fir_bwd_dh_partial_kernel<T>,
                dim3(static_cast<unsigned>(grid)), dim3(hyena::bwd::kDhTaps), smem, s,
                static_cast<const T *>(P.q), static_cast<const T *>(P.k),
                static_cast<const T *>(P.v), static_cast<const T *>(dy), partial, P.L, P.D,
                P.l_h, b.cp, b.nchunk, b.npieces, static_cast<int>(P.B), run_if,
                run_token) != cudaSuccess ||
      cudaGetLastError() != cudaSuccess)
    return HYENA_ERR_CUDA;
  const long long gn = P.G() * P.l_h;  // one warp per output
  long long rblocks = (gn + hyena::bwd::kReduceBlock / 32 - 1) / (hyena::bwd::kReduceBlock / 32);
  if (rblocks > (run_if ? ds->sm_count : cap)) rblocks = run_if ? ds->sm_count : cap;
  if (launch_ex(run_if != nullptr, hyena::bwd::fir_bwd_dh_reduce_kernel,
                dim3(static_cast<unsigned>(rblocks)), dim3(hyena::bwd::kReduceBlock), 0, s,
                static_cast<const float *>(partial), dh, static_cast<int>(P.B), b.nchunk,
                b.npieces, P.d_g / b.cp, static_cast<int>(P.G()), P.l_h, run_if,
                run_token) != cudaSuccess)
    return HYENA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

// Short filters: fir_bwd_window_kernel (dk, dv and a dh partial per thread) and the fixed-order
// reduction of the partials (one piece per channel vector).  The run length follows the
// forward's one-wave rule; it grows where the workspace cannot hold one partial per thread.
template <typename T, int LH>
int launch_window_bwd_lh(const Problem &P, WindowParams wp, const void *dy, void *dk, void *dv,
                         float *dh, float *partial, int64_t partial_floats, int sm_count,
                         cudaStream_t s) {
  const auto kernel = hyena::bwd::fir_bwd_window_kernel<T, LH>;
  static std::atomic<int> resident[kMaxDevices];
  int per_sm = 0;
  if (resident_blocks(kernel, hyena::bwd::kBwdWindowBlock, resident, per_sm) != HYENA_OK)
    return HYENA_ERR_CUDA;
  const long long wave = static_cast<long long>(sm_count) * per_sm * hyena::bwd::kBwdWindowBlock;
  const long long units = wp.B * wp.cv;
  long long rows = window_rows(units, wp.L, wave);
  const long long max_tb = partial_floats / (units * LH);  // time blocks the workspace holds
  if (max_tb < 1) return HYENA_ERR_INVALID_ARG;
  if ((wp.L + rows - 1) / rows > max_tb) rows = (wp.L + max_tb - 1) / max_tb;
  wp.rows = static_cast<int>(rows);
  wp.n_tb = (wp.L + rows - 1) / rows;
  const long long threads = units * wp.n_tb;
  const long long blocks =
      (threads + hyena::bwd::kBwdWindowBlock - 1) / hyena::bwd::kBwdWindowBlock;
  if (blocks > std::numeric_limits<int32_t>::max() || wp.n_tb > std::numeric_limits<int32_t>::max() ||
      wp.cv > std::numeric_limits<int32_t>::max() ||
      wp.B * wp.n_tb * (P.d_g / (wp.D / wp.cv)) > std::numeric_limits<int32_t>::max())
    return HYENA_ERR_UNSUPPORTED;
  if (launch_ex(true, kernel, dim3(static_cast<unsigned>(blocks)),
                dim3(hyena::bwd::kBwdWindowBlock), 0, s, static_cast<const T *>(P.q),
                static_cast<const T *>(P.k), static_cast<const T *>(P.v),
                static_cast<const float *>(P.h), static_cast<const T *>(dy),
                static_cast<T *>(dk), static_cast<T *>(dv), partial, wp) != cudaSuccess ||
      cudaGetLastError() != cudaSuccess)
    return HYENA_ERR_CUDA;
  const long long gn = P.G() * P.l_h;  // one warp per output
  long long rblocks = (gn + hyena::bwd::kReduceBlock / 32 - 1) / (hyena::bwd::kReduceBlock / 32);
  const long long cap = static_cast<long long>(sm_count) * 16;
  if (rblocks > cap) rblocks = cap;
  hyena::bwd::fir_bwd_dh_reduce_kernel<<<static_cast<unsigned>(rblocks),
                                         hyena::bwd::kReduceBlock, 0, s>>>(
      partial, dh, static_cast<int>(P.B), static_cast<int>(wp.n_tb), static_cast<int>(wp.cv),
      static_cast<int>(P.d_g / (wp.D / wp.cv)), static_cast<int>(P.G()), P.l_h, nullptr, 0u);
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

template <typename T, int LH = 1>
int launch_window_bwd_dispatch(const Problem &P, const WindowParams &wp, const void *dy,
                               void *dk, void *dv, float *dh, float *partial,
                               int64_t partial_floats, int sm_count, cudaStream_t s) {
  if constexpr (LH <= kMaxWindowTaps) {
    if (P.l_h == LH)
      return launch_window_bwd_lh<T, LH>(P, wp, dy, dk, dv, dh, partial, partial_floats,
                                         sm_count, s);
    return launch_window_bwd_dispatch<T, LH + 1>(P, wp, dy, dk, dv, dh, partial, partial_floats,
                                                 sm_count, s);
  }
  return HYENA_ERR_UNSUPPORTED;
}

bool window_bwd_supported(const Problem &P, const void *dy, const void *dk, const void *dv) {
  const int vec = P.dtype == HYENA_DTYPE_F32 ? 4 : 8;
  return P.l_h <= kMaxWindowTaps && P.d_g % vec == 0 && aligned(P.q, 16) && aligned(P.k, 16) &&
         aligned(P.v, 16) && aligned(dy, 16) && aligned(dk, 16) && aligned(dv, 16);
}

// dq through the forward kernels (dy in the place of q), then fir_bwd_window_kernel and the
// reduction of its dh partials.
int run_bwd_window(const Problem &P, const void *dy, void *dq, void *dk, void *dv, float *dh,
                   void *workspace, size_t workspace_bytes, cudaStream_t s) {
  Problem F = P;
  F.q = dy;
  F.y = dq;
  const int r = run(F, HYENA_ALGO_AUTO, s);
  if (r != HYENA_OK) return r;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  WindowParams wp{};
  wp.B = P.B;
  wp.L = P.L;
  wp.D = P.D;
  wp.d_g = P.d_g;
  wp.cv = P.D / (P.dtype == HYENA_DTYPE_F32 ? 4 : 8);
  const int64_t floats = static_cast<int64_t>(workspace_bytes / 4);
  float *partial = static_cast<float *>(workspace);
  if (P.dtype == HYENA_DTYPE_F32)
    return launch_window_bwd_dispatch<float>(P, wp, dy, dk, dv, dh, partial, floats,
                                             ds->sm_count, s);
  return launch_window_bwd_dispatch<__nv_bfloat16>(P, wp, dy, dk, dv, dh, partial, floats,
                                                   ds->sm_count, s);
}

// dq through the forward kernels (dy in the place of q), then the CUDA-core dx/dk/dv and dh
// kernels.
int run_bwd_cuda_core(const Problem &P, const void *dy, void *dq, void *dk, void *dv, float *dh,
                      void *workspace, cudaStream_t s) {
  Problem F = P;
  F.q = dy;
  F.y = dq;
  const int r = run(F, HYENA_ALGO_AUTO, s);
  if (r != HYENA_OK) return r;
  if (P.dtype == HYENA_DTYPE_F32)
    return launch_bwd_cuda_core<float>(P, dy, dk, dv, dh, static_cast<float *>(workspace), s);
  return launch_bwd_cuda_core<__nv_bfloat16>(P, dy, dk, dv, dh, static_cast<float *>(workspace),
                                             s);
}

bool tc_bwd_supported(const Problem &P, const void *dy, const void *dq, const void *dk,
                      const void *dv) {
  // the CUDA-core kernels stand behind it for operands outside fp16's range
  return P.dtype == HYENA_DTYPE_BF16 && P.d_g == hyena::tc::kNC && P.D % hyena::tc::kNC == 0 &&
         cuda_core_bwd_launchable(P) && P.l_h <= hyena::tcb::kMaxHalo + 1 &&
         P.L <= (int64_t{1} << 30) &&
         P.B <= (int64_t{1} << 30) && aligned(P.q, 16) && aligned(P.k, 16) &&
         aligned(P.v, 16) && aligned(dy, 16) && aligned(dq, 16) && aligned(dk, 16) &&
         aligned(dv, 16);
}

// dq = dy * (h conv x) is the forward with dy in the place of q (the tuned forward kernel);
// then fir_tc_bwd_kernel (dx, dk, dv and the dh partials) and the fixed-order dh reduction.
int launch_tensor_bwd(const Problem &P, const void *dy, void *dq, void *dk, void *dv, float *dh,
                      void *workspace, size_t workspace_bytes, cudaStream_t s) {
  namespace tb = hyena::tcb;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return HYENA_ERR_CUDA;
  CUtensorMap maps[4];
  const void *ptrs[4] = {P.q, P.k, P.v, dy};
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(P.D), static_cast<cuuint64_t>(P.L),
                              static_cast<cuuint64_t>(P.B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(P.D) * 2,
                                 static_cast<cuuint64_t>(P.L) * static_cast<cuuint64_t>(P.D) * 2};
  const cuuint32_t box[3] = {hyena::tc::kNC, hyena::tc::kTM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  for (int i = 0; i < 4; ++i) {
    if (enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptrs[i]), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            HYENA_TC_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return HYENA_ERR_CUDA;
  }
  tb::Params p;
  p.h = P.h;
  p.B = static_cast<int>(P.B);
  p.L = static_cast<int>(P.L);
  p.l_h = P.l_h;
  p.G = static_cast<int>(P.D / hyena::tc::kNC);
  p.halo = (P.l_h - 1 + 15) / 16 * 16;
  p.band_cols = (hyena::tc::kTM + p.halo) / 2;
  p.nT = static_cast<int>((P.L + hyena::tc::kTM - 1) / hyena::tc::kTM);
  p.W = static_cast<long long>(p.G) * P.B * p.nT;
  int64_t grid = ds->sm_count;
  if (grid > p.W) grid = p.W;
  if (grid > kTcBwdMaxGrid) grid = kTcBwdMaxGrid;
  const int64_t per = p.W / grid;
  p.max_segs = static_cast<int>(per / p.nT + 2);
  const TcBwdLayout lay = tc_bwd_layout(grid * p.max_segs, grid, P.l_h);
  if (lay.bytes > static_cast<int64_t>(workspace_bytes)) return HYENA_ERR_INVALID_ARG;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  p.partial = reinterpret_cast<float *>(ws);
  p.seg_group = reinterpret_cast<int *>(ws + lay.off_group);
  p.seg_count = reinterpret_cast<int *>(ws + lay.off_count);
  p.D = P.D;
  p.dk = static_cast<__nv_bfloat16 *>(dk);
  p.dv = static_cast<__nv_bfloat16 *>(dv);
  const int64_t flag_off = bwd_flag_offset(P.B, P.L, P.D, P.d_g, P.l_h);
  if (flag_off + 4 > static_cast<int64_t>(workspace_bytes)) return HYENA_ERR_INVALID_ARG;
  // The flag word is never reset: the kernel writes this call's token into it, and the fallback
  // kernels run only where they find that token (a stale word from an earlier call, or
  // whatever the workspace held, cannot match; if it ever did, the fp32 kernels would only
  // redo the same gradients).
  static std::atomic<unsigned> tokens{0};
  unsigned token = tokens.fetch_add(1, std::memory_order_relaxed) + 1;
  if (token == 0) token = tokens.fetch_add(1, std::memory_order_relaxed) + 1;
  p.range_flag = reinterpret_cast<unsigned *>(ws + flag_off);
  p.range_token = token;
  Problem F = P;  // dq through the forward kernels
  F.q = dy;
  F.y = dq;
  const int rf = run(F, HYENA_ALGO_AUTO, s);
  if (rf != HYENA_OK) return rf;
  // Programmatic dependent launch: the set-up overlaps the end of the dq forward.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = HYENA_PDL;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(tb::kThreads);
  cfg.dynamicSmemBytes = tb::kSmemBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, tb::fir_tc_bwd_kernel, maps[0], maps[1], maps[2], maps[3], p) !=
          cudaSuccess ||
      cudaGetLastError() != cudaSuccess)
    return HYENA_ERR_CUDA;
  const long long gn = static_cast<long long>(p.G) * P.l_h;
  long long rblocks = (gn + 255) / 256;
  if (rblocks > ds->sm_count) rblocks = ds->sm_count;
  if (launch_ex(true, tb::fir_bwd_tc_reduce_kernel, dim3(static_cast<unsigned>(rblocks)),
                dim3(256), 0, s, static_cast<const float *>(p.partial),
                static_cast<const int *>(p.seg_group), static_cast<const int *>(p.seg_count),
                p.max_segs, dh, p.G, P.l_h, per, static_cast<long long>(p.W % grid),
                static_cast<long long>(P.B) * p.nT) != cudaSuccess ||
      cudaGetLastError() != cudaSuccess)
    return HYENA_ERR_CUDA;
  // Where an fp16 operand left its range (the kernel raised the flag), the fp32 CUDA-core
  // kernels redo dk, dv and dh; otherwise each of them returns at once.
  return launch_bwd_cuda_core<__nv_bfloat16>(P, dy, dk, dv, dh, reinterpret_cast<float *>(ws), s,
                                             p.range_flag, token);
}

// FFT path: N = N1 N2 >= L + l_h - 1 (power of two, >= 256), N1 >= N2, both in [16, 256].
struct FftPlan {
  int N1, N2, log1, log2;
  int64_t N;
  bool ok;
};

FftPlan fft_plan(int64_t L, int l_h) {
  FftPlan f{0, 0, 0, 0, 0, false};
  const int64_t need = L + l_h - 1;
  int m = 8;
  while ((int64_t{1} << m) < need && m < 40) ++m;
  f.log1 = (m + 1) / 2;
  f.log2 = m / 2;
  f.N1 = 1 << f.log1;
  f.N2 = 1 << f.log2;
  f.N = int64_t{1} << m;
  f.ok = f.N1 <= hyena::fft::kMaxLen;
  return f;
}

struct FftLayout {
  int64_t off_hspec, off_h, bytes;
};

// Workspace: the data spectra [B][N1][N2][D/2] complex, the filters' pass-1 output and their
// spectrum [N1 N2][G] complex.
FftLayout fft_layout(int64_t B, int64_t D, int64_t G, int64_t N) {
  FftLayout o;
  o.off_hspec = round256(B * N * (D / 2) * 8);
  o.off_h = o.off_hspec + round256(N * G * 8);
  o.bytes = o.off_h + round256(N * G * 8);
  return o;
}

// 0 when the FFT path takes the shape, else the error it returns.
int fft_supported(const Problem &P, FftPlan &f) {
  if (P.D % 2 != 0 || P.d_g % 2 != 0) return HYENA_ERR_UNSUPPORTED;
  f = fft_plan(P.L, P.l_h);
  const int64_t i32 = std::numeric_limits<int32_t>::max();
  if (!f.ok || P.B > 65535 || (P.D / 2 + hyena::fft::kP - 1) / hyena::fft::kP > 65535 ||
      (P.G() + hyena::fft::kP - 1) / hyena::fft::kP > 65535 || P.L * P.D > i32 ||
      f.N * (P.D / 2) > i32 || f.N * P.G() > i32 || P.G() * static_cast<int64_t>(P.l_h) > i32)
    return HYENA_ERR_UNSUPPORTED;
  return HYENA_OK;
}

template <typename T, int N1>
void launch_fft_p1(const Problem &P, const hyena::fft::FftParams &p, dim3 grid, float2 *A,
                   cudaStream_t s) {
  launch_ex(true, hyena::fft::fft_pass1_kernel<T, false, N1>, grid, dim3(hyena::fft::kThreads), 0,
            s, static_cast<const T *>(P.k), static_cast<const T *>(P.v),
            static_cast<const float *>(nullptr), A, p);
}

template <int N1>
void launch_fft_spec1(const Problem &P, const hyena::fft::FftParams &p, dim3 grid, float2 *A,
                      cudaStream_t s) {
  launch_ex(true, hyena::fft::fft_pass1_kernel<float, true, N1>, grid,
            dim3(hyena::fft::kThreads), 0, s, static_cast<const float *>(nullptr),
            static_cast<const float *>(nullptr), P.h, A, p);
}

template <typename T, int N1>
void launch_fft_p3(const Problem &P, const hyena::fft::FftParams &p, dim3 grid, const float2 *A,
                   cudaStream_t s) {
  launch_ex(true, hyena::fft::fft_pass3_kernel<T, N1>, grid, dim3(hyena::fft::kThreads), 0, s, A,
            static_cast<const T *>(P.q), static_cast<T *>(P.y), p);
}

template <bool kSpectrum, int N2>
void launch_fft_p2(const hyena::fft::FftParams &p, dim3 grid, float2 *A, float2 *H,
                   cudaStream_t s) {
  launch_ex(true, hyena::fft::fft_pass2_kernel<kSpectrum, N2>, grid, dim3(hyena::fft::kThreads), 0,
            s, A, H, p);
}

// Calls F<n>() for the transform length n in {16, ..., 256}.
template <typename F>
bool with_len(int n, F &&f) {
  switch (n) {
    case 16: f(std::integral_constant<int, 16>()); return true;
    case 32: f(std::integral_constant<int, 32>()); return true;
    case 64: f(std::integral_constant<int, 64>()); return true;
    case 128: f(std::integral_constant<int, 128>()); return true;
    case 256: f(std::integral_constant<int, 256>()); return true;
    default: return false;
  }
}

template <typename T>
int launch_fft(const Problem &P, const FftPlan &f, uint8_t *ws, cudaStream_t s) {
  namespace hf = hyena::fft;
  const FftLayout lay = fft_layout(P.B, P.D, P.G(), f.N);
  float2 *A = reinterpret_cast<float2 *>(ws);
  float2 *Hs = reinterpret_cast<float2 *>(ws + lay.off_hspec);
  float2 *Hh = reinterpret_cast<float2 *>(ws + lay.off_h);
  hf::FftParams p;
  p.L = static_cast<int>(P.L);
  p.D = static_cast<int>(P.D);
  p.d_g = P.d_g;
  p.l_h = P.l_h;
  p.N1 = f.N1;
  p.N2 = f.N2;
  p.G = static_cast<int>(P.G());
  const int vec_ch = 16 / static_cast<int>(P.elem());  // channels per 16-byte vector
  p.vec = P.D % vec_ch == 0 && aligned(P.q, 16) && aligned(P.k, 16) && aligned(P.v, 16) &&
          aligned(P.y, 16);
  // the filters' spectrum H[k1][k2][g]
  hf::FftParams ph = p;
  ph.PT = static_cast<int>(P.G());
  const unsigned gb = static_cast<unsigned>((ph.PT + hf::kP - 1) / hf::kP);
  // the data: pass 1, pass 2 (times H, inverse), pass 3 (inverse, q gate)
  p.PT = static_cast<int>(P.D / 2);
  const unsigned db = static_cast<unsigned>((p.PT + hf::kP - 1) / hf::kP);
  const unsigned nb = static_cast<unsigned>(P.B);
  const dim3 g1h(f.N2, gb, 1), g2h(f.N1, gb, 1), g1(f.N2, db, nb), g2(f.N1, db, nb);
  bool ok = with_len(f.N1, [&](auto n1) { launch_fft_spec1<decltype(n1)::value>(P, ph, g1h, Hh, s); });
  ok = ok && with_len(f.N2, [&](auto n2) { launch_fft_p2<true, decltype(n2)::value>(ph, g2h, Hh, Hs, s); });
  ok = ok && with_len(f.N1, [&](auto n1) { launch_fft_p1<T, decltype(n1)::value>(P, p, g1, A, s); });
  ok = ok && with_len(f.N2, [&](auto n2) { launch_fft_p2<false, decltype(n2)::value>(p, g2, A, Hs, s); });
  ok = ok && with_len(f.N1, [&](auto n1) { launch_fft_p3<T, decltype(n1)::value>(P, p, g1, A, s); });
  if (!ok) return HYENA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

// Host checks of a backward call; HYENA_OK, kEmpty or an error code.
int validate_bwd(const Problem &P, const void *dy, void *dq, void *dk, void *dv, float *dh,
                 void *workspace, size_t workspace_bytes) {
  const int rc = validate(P);  // q, k, v, h and dq (in the place of y)
  if (rc == kEmpty) return (!dh || !aligned(dh, 4)) ? HYENA_ERR_INVALID_ARG : kEmpty;
  if (rc != HYENA_OK) return rc;
  if (!dy || !dk || !dv || !dh) return HYENA_ERR_INVALID_ARG;
  const uintptr_t es = static_cast<uintptr_t>(P.elem());
  if (!aligned(dy, es) || !aligned(dk, es) || !aligned(dv, es) || !aligned(dh, 4) ||
      !aligned(workspace, 16))
    return HYENA_ERR_MISALIGNED;
  const int64_t bytes = P.numel() * P.elem();
  const void *ins[] = {P.q, P.k, P.v, dy};
  const void *outs[] = {dq, dk, dv};
  for (int i = 0; i < 3; ++i) {
    for (const void *in : ins)
      if (overlaps(outs[i], in, bytes)) return HYENA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], outs[j], bytes)) return HYENA_ERR_INVALID_ARG;
  }
  if (!workspace ||
      static_cast<int64_t>(workspace_bytes) < bwd_required_bytes(P.B, P.L, P.D, P.d_g, P.l_h))
    return HYENA_ERR_INVALID_ARG;
  return HYENA_OK;
}

// The backward algorithm: HYENA_ALGO_TENSOR (fused tcgen05 kernel) or HYENA_ALGO_DIRECT
// (CUDA-core kernels, dq through the forward), or minus HYENA_ERR_UNSUPPORTED.
int select_bwd(const Problem &P, const void *dy, const void *dq, const void *dk, const void *dv,
               int algo) {
  const bool tc = tc_bwd_supported(P, dy, dq, dk, dv);
  const bool win = window_bwd_supported(P, dy, dk, dv);
  switch (algo) {
    case HYENA_ALGO_AUTO:
      return tc ? HYENA_ALGO_TENSOR : (win ? HYENA_ALGO_WINDOW : HYENA_ALGO_DIRECT);
    case HYENA_ALGO_TENSOR: return tc ? HYENA_ALGO_TENSOR : -HYENA_ERR_UNSUPPORTED;
    case HYENA_ALGO_WINDOW: return win ? HYENA_ALGO_WINDOW : -HYENA_ERR_UNSUPPORTED;
    case HYENA_ALGO_DIRECT: return HYENA_ALGO_DIRECT;
    case HYENA_ALGO_FFT: return -HYENA_ERR_UNSUPPORTED;  // a forward-only algorithm
    default: return -HYENA_ERR_INVALID_ARG;
  }
}

int run_bwd(const Problem &P, const void *dy, void *dq, void *dk, void *dv, float *dh,
            void *workspace, size_t workspace_bytes, cudaStream_t s, int algo) {
  const int rc = validate_bwd(P, dy, dq, dk, dv, dh, workspace, workspace_bytes);
  if (rc == kEmpty)  // no tokens: dh is an empty sum
    return cudaMemsetAsync(dh, 0, static_cast<size_t>(P.G() * P.l_h) * 4, s) == cudaSuccess
               ? HYENA_OK
               : HYENA_ERR_CUDA;
  if (rc != HYENA_OK) return rc;
  const int a = select_bwd(P, dy, dq, dk, dv, algo);
  if (a < 0) return -a;
  if (a == HYENA_ALGO_TENSOR)
    return launch_tensor_bwd(P, dy, dq, dk, dv, dh, workspace, workspace_bytes, s);
  if (a == HYENA_ALGO_WINDOW)
    return run_bwd_window(P, dy, dq, dk, dv, dh, workspace, workspace_bytes, s);
  return run_bwd_cuda_core(P, dy, dq, dk, dv, dh, workspace, s);
}


}  // namespace

// Partials of hyena_conv_bwd_static_scratch: a fixed device array instead of a caller workspace,
// for callers that cannot allocate device memory (see the header).  Every partial the dh kernel
// reads is written earlier in the same call, so nothing in it has to start at zero.
static __device__ __align__(256) float g_bwd_static_scratch[HYENA_BWD_STATIC_SCRATCH_BYTES / 4];

namespace {

struct StaticScratch {
  std::mutex mu;
  void *ptr = nullptr;  // null until a lookup succeeded
};
StaticScratch g_static_scratch[kMaxDevices];

// The current device's address of g_bwd_static_scratch.  The first successful lookup (with
// that device current) is kept for the device; a failed one is not kept, so the next call
// tries again.
int static_scratch(void *&ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HYENA_ERR_CUDA;
  StaticScratch *sc = &g_static_scratch[dev];
  std::lock_guard<std::mutex> lock(sc->mu);
  if (!sc->ptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // clear it, so that a later launch check does not report it
      return HYENA_ERR_CUDA;
    }
    sc->ptr = p;
  }
  ptr = sc->ptr;
  return HYENA_OK;
}

}  // namespace

// ------------------------------------------------------------------------------ from host
// hyena_conv_fwd_from_host: the forward of host-resident q, k, v, h into host y.  Each
// sequence is cut into chunks of `chunk` rows; chunk [t0, t1) travels to the device with the
// l_h - 1 rows before it (rows [s0, t1), s0 = max(0, t0 - l_h + 1)), is computed as a sequence
// of its own (rows from t0 on then equal the whole sequence's), and rows [t0, t1) come back.
// Three device slots rotate over three streams (copy in, compute, copy out) so that the
// host-to-device copy of one chunk, the kernel of the previous one and the copy back of the one
// before overlap (PCIe is full duplex).
constexpr int kHostSlots = 3;

struct HostPipe {
  std::once_flag once;
  std::mutex mu;  // one call at a time per device: the streams and events are shared
  cudaError_t err = cudaSuccess;
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, loaded[kHostSlots] = {}, done[kHostSlots] = {},
              freed[kHostSlots] = {}, tail_in = nullptr, tail_comp = nullptr, finish = nullptr;
};
HostPipe g_host_pipes[kMaxDevices];

struct HostLayout {
  int64_t rows, slot_bytes, off_h, bytes;
};

// Device workspace: kHostSlots slots of (q, k, v, y) chunk buffers, then h.
HostLayout host_layout(int64_t L, int64_t D, int64_t G, int l_h, int64_t elem, int64_t chunk) {
  HostLayout o;
  o.rows = std::min(L, chunk) + l_h - 1;
  o.slot_bytes = 4 * round256(o.rows * D * elem);
  o.off_h = kHostSlots * o.slot_bytes;
  o.bytes = o.off_h + round256(G * l_h * 4);
  return o;
}

int host_pipe(HostPipe *&hp) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HYENA_ERR_CUDA;
  hp = &g_host_pipes[dev];
  HostPipe *h = hp;
  std::call_once(h->once, [h]() {
    cudaError_t e = cudaSuccess;
    for (cudaStream_t *st : {&h->in, &h->comp, &h->out})
      if (e == cudaSuccess) e = cudaStreamCreateWithFlags(st, cudaStreamNonBlocking);
    const unsigned fl = cudaEventDisableTiming;
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->start, fl);
    for (cudaEvent_t *ev : {&h->finish, &h->tail_in, &h->tail_comp})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, fl);
    for (int i = 0; i < kHostSlots && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&h->loaded[i], fl);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->done[i], fl);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->freed[i], fl);
      // a recorded "freed" event lets the first chunk of every slot wait on it unconditionally
      if (e == cudaSuccess) e = cudaEventRecord(h->freed[i], h->out);
    }
    h->err = e;
  });
  return h->err == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

int fwd_from_host(const Problem &P, int64_t chunk, void *workspace, size_t workspace_bytes,
                  cudaStream_t stream) {
  const int64_t es = P.elem(), D = P.D, hist = P.l_h - 1;
  const HostLayout lay = host_layout(P.L, D, P.G(), P.l_h, es, chunk);
  if (!workspace || static_cast<int64_t>(workspace_bytes) < lay.bytes) return HYENA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return HYENA_ERR_MISALIGNED;
  DeviceState *ds = nullptr;
  HostPipe *hp = nullptr;
  if (current_device(ds) != HYENA_OK || host_pipe(hp) != HYENA_OK) return HYENA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->mu);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *hd = reinterpret_cast<float *>(ws + lay.off_h);
  const int64_t tensor_bytes = round256(lay.rows * D * es);
  const uint8_t *src[3] = {static_cast<const uint8_t *>(P.q), static_cast<const uint8_t *>(P.k),
                           static_cast<const uint8_t *>(P.v)};
  uint8_t *yh = static_cast<uint8_t *>(P.y);
  cudaError_t e = cudaEventRecord(hp->start, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->in, hp->start, 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(hd, P.h, static_cast<size_t>(P.G() * P.l_h * 4), cudaMemcpyHostToDevice,
                        hp->in);
  int64_t n = 0;
  int status = HYENA_OK;
  for (int64_t b = 0; b < P.B && e == cudaSuccess && status == HYENA_OK; ++b) {
    for (int64_t t0 = 0; t0 < P.L && e == cudaSuccess; t0 += chunk, ++n) {
      const int64_t t1 = std::min(P.L, t0 + chunk), s0 = std::max<int64_t>(0, t0 - hist);
      const int64_t nr = t1 - s0, nh = t0 - s0;  // rows in the slot, of which history
      const int si = static_cast<int>(n % kHostSlots);
      uint8_t *slot = ws + si * lay.slot_bytes;
      uint8_t *dev[4] = {slot, slot + tensor_bytes, slot + 2 * tensor_bytes,
                         slot + 3 * tensor_bytes};
      const size_t row_bytes = static_cast<size_t>(D * es), hbytes = nh * row_bytes;
      const size_t nbytes = static_cast<size_t>(t1 - t0) * row_bytes;
      const int64_t row0 = (b * P.L + t0) * D * es;
      // copy in once the slot's previous chunk has been copied out: rows [t0, t1) from the
      // host; the history rows of k and v from the previous chunk's slot (already on the device,
      // queued earlier on the same stream); the history rows of q only feed outputs that are
      // dropped, so they are zeroed
      e = cudaStreamWaitEvent(hp->in, hp->freed[si], 0);
      for (int i = 0; i < 3 && e == cudaSuccess; ++i)
        e = cudaMemcpyAsync(dev[i] + hbytes, src[i] + row0, nbytes, cudaMemcpyHostToDevice,
                            hp->in);
      if (nh > 0 && e == cudaSuccess) {
        // the previous chunk of this sequence (t0 > 0) sits in slot n - 1, its rows from s0p
        const int sp = static_cast<int>((n + kHostSlots - 1) % kHostSlots);
        const int64_t s0p = std::max<int64_t>(0, t0 - chunk - hist);
        uint8_t *prev = ws + sp * lay.slot_bytes;
        const size_t off = static_cast<size_t>(s0 - s0p) * row_bytes;
        e = cudaMemsetAsync(dev[0], 0, hbytes, hp->in);
        for (int i = 1; i < 3 && e == cudaSuccess; ++i)
          e = cudaMemcpyAsync(dev[i], prev + i * tensor_bytes + off, hbytes,
                              cudaMemcpyDeviceToDevice, hp->in);
      }
      if (e == cudaSuccess) e = cudaEventRecord(hp->loaded[si], hp->in);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->comp, hp->loaded[si], 0);
      if (e != cudaSuccess) break;
      Problem C = P;
      C.q = dev[0];
      C.k = dev[1];
      C.v = dev[2];
      C.y = dev[3];
      C.h = hd;
      C.B = 1;
      C.L = nr;
      status = run(C, HYENA_ALGO_AUTO, hp->comp);
      if (status != HYENA_OK) break;
      e = cudaEventRecord(hp->done[si], hp->comp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->out, hp->done[si], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(yh + (b * P.L + t0) * D * es, dev[3] + (t0 - s0) * D * es,
                            static_cast<size_t>((t1 - t0) * D * es), cudaMemcpyDeviceToHost,
                            hp->out);
      if (e == cudaSuccess) e = cudaEventRecord(hp->freed[si], hp->out);
    }
  }
  // `stream` waits for everything queued on the three streams, also after an error, so that
  // synchronising it covers every copy that still reads the caller's buffers
  cudaError_t t = cudaEventRecord(hp->tail_in, hp->in);
  if (t == cudaSuccess) t = cudaEventRecord(hp->tail_comp, hp->comp);
  if (t == cudaSuccess) t = cudaStreamWaitEvent(hp->out, hp->tail_in, 0);
  if (t == cudaSuccess) t = cudaStreamWaitEvent(hp->out, hp->tail_comp, 0);
  if (t == cudaSuccess) t = cudaEventRecord(hp->finish, hp->out);
  if (t == cudaSuccess) t = cudaStreamWaitEvent(stream, hp->finish, 0);
  if (status != HYENA_OK) return status;
  return e == cudaSuccess && t == cudaSuccess && cudaGetLastError() == cudaSuccess
             ? HYENA_OK
             : HYENA_ERR_CUDA;
}

extern "C" {

int hyena_conv_fwd(const void *q, const void *k, const void *v, const float *h, void *y,
                   int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                   cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, HYENA_DTYPE_BF16};
  return run(P, HYENA_ALGO_AUTO, stream);
}

int hyena_conv_fwd_f32(const float *q, const float *k, const float *v, const float *h, float *y,
                       int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                       cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, HYENA_DTYPE_F32};
  return run(P, HYENA_ALGO_AUTO, stream);
}

int hyena_conv_fwd_ex(const void *q, const void *k, const void *v, const float *h, void *y,
                      int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype,
                      int algo, cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, dtype};
  return run(P, algo, stream);
}

int hyena_conv_fwd_hist(const void *q, const void *k, const void *v, const float *h, void *y,
                        const void *k_hist, const void *v_hist, int64_t L_hist, int64_t B,
                        int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype, int algo,
                        cudaStream_t stream) {
  if (L_hist < 0) return HYENA_ERR_INVALID_ARG;
  Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, dtype};
  P.kh = k_hist;
  P.vh = v_hist;
  P.Lh = L_hist;
  return run(P, algo, stream);
}

int64_t hyena_conv_fwd_fft_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1) return -HYENA_ERR_INVALID_ARG;
  const Problem P{nullptr, nullptr, nullptr, nullptr, nullptr, B, L, D, d_g, l_h, 1,
                  HYENA_DTYPE_BF16};
  if (B == 0 || L == 0) return 0;
  FftPlan f{};
  if (fft_supported(P, f) != HYENA_OK) return -HYENA_ERR_UNSUPPORTED;
  return fft_layout(B, D, P.G(), f.N).bytes;
}

int hyena_conv_fwd_fft(const void *q, const void *k, const void *v, const float *h, void *y,
                       int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, dtype};
  const int rc = validate(P);
  if (rc == kEmpty) return HYENA_OK;
  if (rc != HYENA_OK) return rc;
  FftPlan f{};
  const int fs = fft_supported(P, f);
  if (fs != HYENA_OK) return fs;
  if (!workspace) return HYENA_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return HYENA_ERR_MISALIGNED;
  if (static_cast<int64_t>(workspace_bytes) < fft_layout(B, D, P.G(), f.N).bytes)
    return HYENA_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  if (dtype == HYENA_DTYPE_F32) return launch_fft<float>(P, f, ws, stream);
  return launch_fft<__nv_bfloat16>(P, f, ws, stream);
}

int hyena_select_algo(const void *q, const void *k, const void *v, const float *h, const void *y,
                      int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype) {
  const Problem P{q, k, v, h, const_cast<void *>(y), B, L, D, d_g, l_h, l_b, dtype};
  const int rc = validate(P);
  if (rc != HYENA_OK && rc != kEmpty) return -rc;
  return select_algo(P);
}

int64_t hyena_conv_bwd_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h) {
  if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1) return -HYENA_ERR_INVALID_ARG;
  return bwd_workspace_bytes(B, L, D, d_g, l_h);
}

int hyena_conv_bwd(const void *q, const void *k, const void *v, const float *h, const void *dy,
                   void *dq, void *dk, void *dv, float *dh, int64_t B, int64_t L, int64_t D,
                   int d_g, int l_h, int l_b, int dtype, void *workspace, size_t workspace_bytes,
                   cudaStream_t stream) {
  const Problem P{q, k, v, h, dq, B, L, D, d_g, l_h, l_b, dtype};
  return run_bwd(P, dy, dq, dk, dv, dh, workspace, workspace_bytes, stream, HYENA_ALGO_AUTO);
}

int hyena_conv_bwd_ex(const void *q, const void *k, const void *v, const float *h,
                      const void *dy, void *dq, void *dk, void *dv, float *dh, int64_t B,
                      int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype, int algo,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  const Problem P{q, k, v, h, dq, B, L, D, d_g, l_h, l_b, dtype};
  return run_bwd(P, dy, dq, dk, dv, dh, workspace, workspace_bytes, stream, algo);
}

int hyena_select_bwd_algo(const void *q, const void *k, const void *v, const float *h,
                          const void *dy, const void *dq, const void *dk, const void *dv,
                          int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                          int dtype) {
  const Problem P{q, k, v, h, const_cast<void *>(dq), B, L, D, d_g, l_h, l_b, dtype};
  const int rc = validate(P);
  if (rc != HYENA_OK && rc != kEmpty) return -rc;
  return select_bwd(P, dy, dq, dk, dv, HYENA_ALGO_AUTO);
}

int hyena_conv_bwd_static_scratch(const void *q, const void *k, const void *v, const float *h,
                                  const void *dy, void *dq, void *dk, void *dv, float *dh,
                                  int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                                  int dtype, cudaStream_t stream) {
  const Problem P{q, k, v, h, dq, B, L, D, d_g, l_h, l_b, dtype};
  const int rc = validate(P);
  if (rc != HYENA_OK && rc != kEmpty) return rc;
  if (rc == HYENA_OK &&
      bwd_required_bytes(B, L, D, d_g, l_h) > static_cast<int64_t>(HYENA_BWD_STATIC_SCRATCH_BYTES))
    return HYENA_ERR_UNSUPPORTED;
  void *ws = nullptr;
  if (static_scratch(ws) != HYENA_OK) return HYENA_ERR_CUDA;
  return run_bwd(P, dy, dq, dk, dv, dh, ws, HYENA_BWD_STATIC_SCRATCH_BYTES, stream,
                 HYENA_ALGO_AUTO);
}

int hyena_testing_fwd_fault(const void *q, const void *k, const void *v, const float *h, void *y,
                            int64_t B, int64_t L, int64_t D, int d_g, int l_h, int fault,
                            uint64_t wait_ns, cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, 1, HYENA_DTYPE_BF16};
  const int rc = validate(P);
  if (rc == kEmpty) return HYENA_OK;
  if (rc != HYENA_OK) return rc;
  if ((fault != 0 && fault != 1) || wait_ns < 1000000ull || wait_ns > hyena::kWaitTimeoutNs)
    return HYENA_ERR_INVALID_ARG;
  if (!tensor_supported(P)) return HYENA_ERR_UNSUPPORTED;
  TcTestHooks hooks;
  hooks.wait_ns = wait_ns;
  hooks.fault = fault;
  return launch_tensor(P, stream, hooks);
}

int hyena_build_toeplitz(const float *h, float *H0, float *H1, float *H2_or_null, int G,
                         int l_h, int l_b, cudaStream_t stream) {
  if (!h || !H0 || !H1 || G < 1 || l_h < 1 || l_b < 1) return HYENA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(l_h) > 2 * static_cast<int64_t>(l_b)) return HYENA_ERR_INVALID_ARG;
  if (l_h >= l_b + 2 && !H2_or_null) return HYENA_ERR_INVALID_ARG;
  if (!aligned(h, 4) || !aligned(H0, 4) || !aligned(H1, 4) || !aligned(H2_or_null, 4))
    return HYENA_ERR_MISALIGNED;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  const long long n = static_cast<long long>(G) * l_b * l_b;
  long long blocks = (n + 255) / 256;
  const long long cap = static_cast<long long>(ds->sm_count) * 8;
  if (blocks > cap) blocks = cap;
  hyena::cc::toeplitz_blocks_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      h, H0, H1, H2_or_null, G, l_h, l_b);
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

int hyena_toeplitz_stages(int l_h, int l_b) {
  if (l_h < 1 || l_b < 1) return -HYENA_ERR_INVALID_ARG;
  return 1 + static_cast<int>((static_cast<int64_t>(l_h) - 1 + l_b - 1) / l_b);
}

int hyena_build_toeplitz_blocks(const float *h, float *Hm, int S, int G, int l_h, int l_b,
                                cudaStream_t stream) {
  if (!h || !Hm || S < 1 || G < 1 || l_h < 1 || l_b < 1) return HYENA_ERR_INVALID_ARG;
  const int64_t sg = static_cast<int64_t>(S) * G, blk = static_cast<int64_t>(l_b) * l_b;
  if (blk > std::numeric_limits<int64_t>::max() / 8 / sg) return HYENA_ERR_INVALID_ARG;
  const int64_t n = sg * blk;
  if (!aligned(h, 4) || !aligned(Hm, 4)) return HYENA_ERR_MISALIGNED;
  DeviceState *ds = nullptr;
  if (current_device(ds) != HYENA_OK) return HYENA_ERR_CUDA;
  long long blocks = (n + 255) / 256;
  const long long cap = static_cast<long long>(ds->sm_count) * 8;
  if (blocks > cap) blocks = cap;
  hyena::cc::toeplitz_stack_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      h, Hm, S, G, l_h, l_b);
  return cudaGetLastError() == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

int hyena_device_status(unsigned int *out, int clear) {
  if (!out) return HYENA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return HYENA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(out, hyena::g_device_status, sizeof(unsigned int)) != cudaSuccess)
    return HYENA_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(hyena::g_device_status, &zero, sizeof(unsigned int)) != cudaSuccess)
      return HYENA_ERR_CUDA;
  }
  return HYENA_OK;
}

const char *hyena_status_string(int status) {
  switch (status) {
    case HYENA_OK:
      return "ok";
    case HYENA_ERR_INVALID_ARG:
      return "invalid argument";
    case HYENA_ERR_UNSUPPORTED:
      return "unsupported shape or alignment for the requested algorithm";
    case HYENA_ERR_MISALIGNED:
      return "pointer not aligned to its element size";
    case HYENA_ERR_CUDA:
      return "CUDA runtime error";
    default:
      return "unknown status";
  }
}

int hyena_abi_version(void) { return 1; }

int64_t hyena_conv_fwd_from_host_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g,
                                                 int l_h, int dtype, int64_t chunk) {
  if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1 || chunk < 1 ||
      (dtype != HYENA_DTYPE_BF16 && dtype != HYENA_DTYPE_F32))
    return -HYENA_ERR_INVALID_ARG;
  if (B == 0 || L == 0) return 0;
  const int64_t es = dtype == HYENA_DTYPE_F32 ? 4 : 2;
  return host_layout(L, D, D / d_g, l_h, es, chunk).bytes;
}

int hyena_conv_fwd_from_host(const void *q, const void *k, const void *v, const float *h,
                             void *y, int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                             int dtype, int64_t chunk, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  const Problem P{q, k, v, h, y, B, L, D, d_g, l_h, l_b, dtype};
  const int rc = validate(P);  // shapes, null pointers, element alignment, y against the inputs
  if (rc == kEmpty) return HYENA_OK;
  if (rc != HYENA_OK) return rc;
  if (chunk < 1) return HYENA_ERR_INVALID_ARG;
  return fwd_from_host(P, chunk, workspace, workspace_bytes, stream);
}

}  // extern "C"
