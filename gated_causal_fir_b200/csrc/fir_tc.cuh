// fir_tc.cuh -- tcgen05 tensor-core kernel of the gated grouped causal FIR (bf16 I/O).
//
// Method: the block-Toeplitz form of the causal FIR (StripedHyena 2 page "04. Hardware-aware
// convolution kernels", Sec. 2 block convolution and Sec. 3 two-stage algorithm,
// Yhat_n = H0 Xhat_n + H1 Xhat_{n-1}, Xhat_{-1} = 0), with the Sec. 4 reuse (the Toeplitz
// operand of a group is built once on chip and reused for every chunk and every channel of the
// group, which turns the per-channel products into one GEMM) and the Sec. 6 chunk-direction
// schedule (each CTA walks consecutive chunks and keeps the previous chunk's input on chip).
//
// One tile = 128 output rows x 64 channels (64 / d_g groups).  The block size of the
// decomposition is 128 rows, the largest M of one tcgen05.mma.  A tile reads its own 128 input
// rows and halo = roundup16(l_h - 1) rows before them, which lie in the kNH = ceil(halo / 128)
// earlier tiles (one for l_h <= 129, where this is the two-stage form of Sec. 3; up to five for
// l_h <= 641, the general block form of Sec. 2; five hold one band set in tensor memory and two
// k/v stages).  As one GEMM per tile and group:
//   D[128 x d_g] = A[128 x K] * X[K x d_g],  K = 128 + halo,
// A is the Toeplitz band over input rows [t0 - halo, t0 + 128), X = k*v over those rows.
//
// B200 specifics:
//  * q, k, v tiles arrive by TMA (128-byte swizzle) into a multi-stage ring; y leaves by TMA
//    store.  The gate warps turn each time-major k, v tile into fp16 X^T (channels as rows,
//    K-major, 128-byte swizzle) with ldmatrix / stmatrix.trans: the B operand of tcgen05.
//  * The band lives in tensor memory (A operand of tcgen05.mma read from TMEM), written once
//    per sequence run by the gate warps with tcgen05.st: output rows are reversed (TMEM lane p
//    holds time t0 + 127 - p), so lane p's row is A[p][kk] = h[127 + halo - p - kk].
//  * Accumulators live in TMEM (2 x 64 columns); the epilogue reads them with tcgen05.ld,
//    multiplies by q and rounds to bf16 in registers, and writes y over the q tile in place.
//  * Warp roles: 0 TMA producer of k and v, 10 TMA producer of q, 1 MMA issuer (+ TMEM
//    owner), 2-5 pre-gate / operand build, 6-9 epilogue.  Persistent grid: one CTA per SM, each
//    walks a contiguous range of tiles ordered (group, batch, time), so halo tiles are re-read
//    only where a range starts inside a sequence.
//  * Launched with programmatic stream serialisation: barrier set-up and the TMEM allocation
//    overlap the previous kernel; nothing global is read before griddepcontrol.wait.
//  * Every wait is bounded (ptx.cuh); a timeout raises HYENA_DEVICE_TIMEOUT, all roles leave
//    their loops, in-flight copies and MMAs are drained and TMEM is freed before exit.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>
#include "ptx.cuh"

namespace hyena {

__device__ unsigned int g_device_status;  // OR of hyena_device_status_bits

namespace tc {

constexpr int kTM = 128;             // output rows per tile (MMA M)
constexpr int kNC = 64;              // channels per tile: 64 / d_g groups of d_g (MMA N = d_g)
constexpr int kMaxHist = 5;          // history tiles a tile may read: l_h - 1 <= 5 * 128
constexpr int kMaxHalo = kMaxHist * kTM;
#ifndef HYENA_TC_KV_STAGES
#define HYENA_TC_KV_STAGES 3
#endif
constexpr int kNKV = HYENA_TC_KV_STAGES;  // k/v stages (two where five history tiles are held)
// Unrolling of the gate's and the epilogue's per-tile loops (8 iterations each).  The kernel's
// warp roles run different code side by side, so hot-loop code size competes for the
// instruction cache.
#ifndef HYENA_TC_GATE_UNROLL
#define HYENA_TC_GATE_UNROLL 8
#endif
#ifndef HYENA_TC_EPI_UNROLL
#define HYENA_TC_EPI_UNROLL 8
#endif
constexpr int kGateUnroll = HYENA_TC_GATE_UNROLL;
constexpr int kEpiUnroll = HYENA_TC_EPI_UNROLL;
constexpr int kNAcc = 2;             // TMEM accumulator sets (tiles in flight)
constexpr int kRowBytes = kNC * 2;                              // 128 B
constexpr int kTileBytes = kTM * kRowBytes;                     // 16 KB
constexpr int kKBlockBytes = kNC * 128;                         // 64 times x 64 channels
// Tensor memory: accumulators in columns [0, kNAcc * 64) (group gg of a tile in columns
// [gg d_g, (gg+1) d_g) of its set); then `nbuf` sets of Toeplitz bands, one band per group of the
// tile, each 128 lanes x band_cols columns = 128 rows x 2 band_cols fp16 K elements, with
// band_cols = (128 + halo) / 2.  The host picks nbuf (2, else 1) so that everything fits.
constexpr int kBandCol0 = kNAcc * kNC;                           // 128
constexpr int kTmemCols = 512;

constexpr int kThreads = 384;
// Limit of the recomputation warp's wait, which spans the whole kernel.
constexpr uint64_t kFixWaitNs = 20000000000ull;  // 20 s
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpGate0 = 2, kWarpEpi0 = 6, kWarpTmaQ = 10,
              kWarpFix = 11;
constexpr int kGroupThreads = 128;

// Shared-memory layout for a kernel whose tiles read kNH earlier tiles (halo <= 128 kNH rows):
// k/v stages, q stages (reused in place for y), and kNH + 2 fp16 X slots (the kNH tiles of
// history, the current tile and the next one being gated).
template <int kNH>
struct Layout {
  static constexpr int kNKV = kNH >= 5 ? 2 : tc::kNKV;  // k/v stages
  static constexpr int kNQ = kNH >= 4 ? 2 : 3;   // q (and in-place y) stages
  static constexpr int kNX = kNH + 2;            // fp16 X slots
  static constexpr int kOffKV = 0;
  static constexpr int kOffQ = kOffKV + kNKV * 2 * kTileBytes;
  static constexpr int kOffX = kOffQ + kNQ * kTileBytes;
  // fp16 filter taps of the tile's groups, zero-padded: 258 + halo per group (see stage_taps);
  // kPer of them per gate thread
  static constexpr int kHzBytes =
      kNH == 1 ? 2688 : (kNH == 2 ? 2064 : (kNH == 3 ? 1296 : (kNH == 4 ? 1552 : 1808)));
  static constexpr int kPer = (kHzBytes / 2 + kGroupThreads - 1) / kGroupThreads;
  static constexpr int kOffHz = kOffX + kNX * kTileBytes;
  // Output tiles whose fp16 operands left the range, listed by the gate warps for the
  // epilogue's fp32 recomputation after its main loop: a count, then up to kNBad walk positions
  // (more than kNBad: every output tile of the CTA is recomputed).
  static constexpr int kNBad = kNH <= 2 ? 8 : 4;
  static constexpr int kOffBad = kOffHz + kHzBytes;
  // Scale exponents of the sequence run, from the gate to the epilogue (two, by run parity):
  // byte gg = eh + ex of the tile's group gg.
  static constexpr int kOffSeg = kOffBad + 8 + kNBad * 8;
  // Per-segment maxima (two sets, by segment parity): |h| of each group (4 words) and |k v| of
  // the segment's first tile (1 word), as float bits.
  static constexpr int kOffMax = kOffSeg + 8;
  static constexpr int kOffBar = kOffMax + 2 * 8 * 4;
  // barriers
  static constexpr int kBarKVFull = 0;
  static constexpr int kBarKVEmpty = kBarKVFull + kNKV;
  static constexpr int kBarQFull = kBarKVEmpty + kNKV;
  static constexpr int kBarQEmpty = kBarQFull + kNQ;
  static constexpr int kBarYReady = kBarQEmpty + kNQ;
  static constexpr int kBarXFull = kBarYReady + kNQ;
  static constexpr int kBarXEmpty = kBarXFull + kNX;
  static constexpr int kBarAccFull = kBarXEmpty + kNX;
  static constexpr int kBarAccEmpty = kBarAccFull + kNAcc;
  static constexpr int kBarAFull = kBarAccEmpty + kNAcc;
  static constexpr int kBarAEmpty = kBarAFull + 2;  // up to two band sets
  static constexpr int kBarGate = kBarAEmpty + 2;   // the 128 gate threads among themselves
  static constexpr int kBarDone = kBarGate + 1;
  static constexpr int kBarSegFull = kBarDone + 1;       // two, by run parity
  static constexpr int kBarSegEmpty = kBarSegFull + 2;
  static constexpr int kBarGateDone = kBarSegEmpty + 2;  // the gate warps have left their loop
  static constexpr int kBarEpiDone = kBarGateDone + 1;   // the epilogue has finished (and, when
                                                         // tiles were listed, its stores landed)
  static constexpr int kNumBars = kBarEpiDone + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget of one CTA exceeded");
};


constexpr unsigned kTimeoutBit = 1u;  // HYENA_DEVICE_TIMEOUT
constexpr unsigned kF16RangeBit = 2u; // HYENA_DEVICE_F16_RANGE

// fp16 operands with power-of-two scales, chosen per sequence run.  The band holds
// fp16(h * 2^eh): eh = 0 while the group's largest |h| lies in [2^-4, 2^8) (fp16 holds such
// taps as they are: a tap far below the largest one keeps an absolute error of at most 2^-25,
// negligible beside it), else the eh that brings it to [2^7, 2^8).  X holds fp16(k v 2^ex) with
// ex chosen from the run's first tile: ex = -eh of the tile's first group whenever that puts
// the tile's largest |k v| in [2^-6, 2^9) (room for later tiles up to 2^7 times larger), so
// that the product needs no rescaling; otherwise the ex that brings it to [2^8, 2^9).  Scaling
// by a power of two is exact, so the accumulator is the unscaled sum times 2^(eh + ex), which
// the epilogue divides out exactly.  For operands of ordinary size eh = ex = 0, and the hot
// loops carry no scaling; the scaled conversions run out of line.  A tile whose inputs still leave
// the range (a scaled |k v| above 65504, or a warp's 32 rows all below 2^-12 but not all
// zero, where most values would be fp16 subnormals) is recomputed in fp32 on the CUDA cores
// once the CTA's stores have landed, and rewritten.
// A value below fp16's normal range (2^-14 scaled) keeps an absolute error of at most 2^-25
// scaled, 2^-(25 + ex) unscaled.
constexpr int kTapExpTarget = 7;
constexpr int kXExpTarget = 8;
constexpr int kXBalancedLo = -6, kXBalancedHi = 8;  // accepted floor(log2 max |k v 2^ex|)
constexpr uint32_t kXTinyBits = 0x39800000u;  // 2^-12 as float bits
constexpr uint32_t kF16MaxBits = 0x477FE000u;  // 65504 as float bits

struct Params {
  const float *h;   // [D / d_g, l_h]
  // the tensors as raw pointers, for the fp32 recomputation of out-of-range tiles
  const __nv_bfloat16 *q, *k, *v, *kh, *vh;
  __nv_bfloat16 *y;
  long long D;      // channels (row length)
  unsigned long long wait_ns;  // limit of the bounded waits between roles
  int fault;        // test hook: 1 = the MMA issuer withholds the first accumulator arrive
  int B, L, l_h;
  int CB;           // 64-channel blocks across D (tiles per time row) = D / 64
  int halo;         // multiple of 16, >= l_h - 1, <= 128 * (history tiles of the kernel)
  int band_cols;    // TMEM columns of one group's band = (128 + halo) / 2
  int nbuf;         // band sets in TMEM (1 or 2)
  int nT;           // tiles per sequence = ceil(L / kTM)
  long long W;      // tiles of the walk: CB * B * nT, or (CB / 2) * B * nT when paired
  int paired;       // CTAs 2p and 2p+1 walk the same (block pair, batch, time) range, one
                    // block each, so both halves of every 256-byte row are read together
  int hist_tiles;   // 0: zero history before row 0; kNH: the rows before row 0 come from the
                    // history tensors (tile i < 0 = their rows Lh + 128 i .. Lh + 128 i + 127)
  int Lh;           // rows of the history tensors
};

// One unit of a CTA's walk: a halo tile (input only) or an output tile.
struct Item {
  int g, b, i;      // 64-channel block, sequence, tile index along time (< 0: history tile)
  int seg;          // running segment number within this CTA (a segment = one sequence run)
  bool halo;        // input-only tile feeding the first output tiles of a segment
  bool last;        // last output tile of its segment
};

// The walk of one CTA: tiles [w_begin, w_end) of the order (group, batch, time); with gmul = 2
// the walk is over group pairs and this CTA takes group 2 * pair + goff.  A segment that starts
// at tile i of a sequence is preceded by its min(i + hist_tiles, nh) history tiles as halo
// items (input only; tiles with i < 0 come from the history tensors).  The position is decoded once; next() only increments (64-bit divisions are software
// routines on the GPU).
struct WorkIter {
  long long w, w_end;
  int nT, B, seg, gmul, nh, hist, hpend, i, g, b;
  bool at_begin, entered;
  __device__ WorkIter(long long w_begin, long long w_end_, int nT_, int B_, int gmul_, int goff,
                      int nh_, int hist_tiles)
      : w(w_begin), w_end(w_end_), nT(nT_), B(B_), seg(-1), gmul(gmul_), nh(nh_),
        hist(hist_tiles), hpend(0), at_begin(true), entered(false) {
    const long long seq = w_begin / nT;
    i = static_cast<int>(w_begin - seq * nT);
    g = static_cast<int>(seq / B) * gmul + goff;
    b = static_cast<int>(seq % B);
  }
  __device__ bool next(Item &it) {
    if (w >= w_end) return false;
    it.g = g;
    it.b = b;
    if ((at_begin || i == 0) && !entered) {
      entered = true;
      ++seg;
      hpend = min(i + hist, nh);
    }
    it.seg = seg;
    if (hpend > 0) {
      it.i = i - hpend;
      it.halo = true;
      it.last = false;
      --hpend;
      return true;
    }
    it.i = i;
    it.halo = false;
    it.last = (w + 1 == w_end) || (i + 1 == nT);
    ++w;
    at_begin = false;
    entered = false;
    if (++i == nT) {
      i = 0;
      if (++b == B) {
        b = 0;
        g += gmul;
      }
    }
    return true;
  }
};

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          uint64_t limit_ns = kWaitTimeoutNs) {
  const bool ok = mbar_wait(bar, parity, abort, &g_device_status, kTimeoutBit, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool thread_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                            uint64_t limit_ns = kWaitTimeoutNs) {
  return mbar_wait(bar, parity, abort, &g_device_status, kTimeoutBit, limit_ns);
}

// Drain wait: bounded by time only (ignores the abort flag), for copies this thread issued.
// Always the full limit: a CTA must not exit with a copy into its shared memory in flight.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  int no_abort = 0;
  mbar_wait(bar, parity, &no_abort, &g_device_status, kTimeoutBit);
}

// x = fp16(k * v) for two bf16 lanes packed in a 32-bit word; k*v is exact in fp32.
__device__ __forceinline__ uint32_t gate_pair(uint32_t kw, uint32_t vw, bool &over) {
  const float k0 = __uint_as_float(kw << 16), k1 = __uint_as_float(kw & 0xFFFF0000u);
  const float v0 = __uint_as_float(vw << 16), v1 = __uint_as_float(vw & 0xFFFF0000u);
  const float x0 = k0 * v0, x1 = k1 * v1;
  over |= (fabsf(x0) > 65504.f) | (fabsf(x1) > 65504.f);
  const __half2 hx = __floats2half2_rn(x0, x1);
  return *reinterpret_cast<const uint32_t *>(&hx);
}

// 2^e as a float, for -126 <= e <= 127.
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// The power-of-two exponent that brings a maximum |value| (float bits) to [2^target,
// 2^(target+1)): 0 for an all-zero maximum, clamped to [-60, 60] so that the epilogue's
// combined factor 2^-(eh + ex) is one normal float.  (Operands beyond what the clamp covers
// leave fp16's range and take the fp32 recomputation.)
__device__ __forceinline__ int scale_exp(uint32_t max_bits, int target) {
  if (max_bits == 0) return 0;
  const int e = static_cast<int>((max_bits >> 23) & 0xFFu) - 127;  // floor(log2 max)
  return min(max(target - e, -60), 60);
}

// eh of a group from its largest |h| (see kTapExpTarget); `clamped` is set when the wanted
// exponent lay beyond the clamp (the run's operands then leave fp16's range).
__device__ __forceinline__ int tap_scale_exp(uint32_t max_bits, bool &clamped) {
  const int e = static_cast<int>((max_bits >> 23) & 0xFFu) - 127;
  if (max_bits == 0 || (e >= -4 && e <= 7)) return 0;
  clamped |= (kTapExpTarget - e > 60) | (kTapExpTarget - e < -60);
  return scale_exp(max_bits, kTapExpTarget);
}

// ex of a sequence run from the largest |k v| of its first tile and the first group's eh (see
// kTapExpTarget); `clamped` as above.
__device__ __forceinline__ int x_scale_exp(uint32_t max_bits, int eh0, bool &clamped) {
  const int e = static_cast<int>((max_bits >> 23) & 0xFFu) - 127;
  if (max_bits == 0 || (e - eh0 >= kXBalancedLo && e - eh0 <= kXBalancedHi)) return -eh0;
  clamped |= (kXExpTarget - e > 60) | (kXExpTarget - e < -60);
  return scale_exp(max_bits, kXExpTarget);
}

// x = fp16(k * v * s) for two bf16 lanes packed in a 32-bit word (s = 2^ex when kScaled; k*v
// and k*v*s are exact in fp32); folds |x| (fp32, before the rounding) into the running
// maximum mx, so that an fp16 overflow shows as mx > 65504 and a value that rounds to zero
// still counts.
template <bool kScaled>
__device__ __forceinline__ uint32_t gate_pair_x(uint32_t kw, uint32_t vw, float s, float &mx) {
  const float k0 = __uint_as_float(kw << 16), k1 = __uint_as_float(kw & 0xFFFF0000u);
  const float v0 = __uint_as_float(vw << 16), v1 = __uint_as_float(vw & 0xFFFF0000u);
  float x0 = k0 * v0, x1 = k1 * v1;
  if (kScaled) {
    x0 *= s;
    x1 *= s;
  }
  mx = fmaxf(mx, fmaxf(fabsf(x0), fabsf(x1)));
  const __half2 hx = __floats2half2_rn(x0, x1);
  return *reinterpret_cast<const uint32_t *>(&hx);
}

// X^T of gate warp gw's 32 rows (channel rows, 64 times per 128-byte row, two 8 KB K-blocks per
// tile, 128-byte swizzle) from the time-major k and v tiles: 8 x 8 blocks moved with ldmatrix,
// k*v (times 2^ex when kScaled) formed in fp32, rounded to fp16 and stored transposed with
// stmatrix (both bank-conflict-free).  Returns this lane's largest |x| before the rounding.
template <bool kScaled>
__device__ __forceinline__ float gate_x_tile(uint32_t kbase, uint32_t vbase, uint32_t xbase,
                                             int gw, int lane, float s) {
  const int mat = lane >> 3, rr = lane & 7;
  float mx = 0.f;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bw = it * 4 + mat;
    const int tg = gw * 4 + (bw >> 3), cg = bw & 7;  // 8-time group, 8-channel group
    const uint32_t src = (tg * 8 + rr) * kRowBytes + ((cg ^ rr) << 4);
    uint32_t kf[4], vf[4], xf[4];
    ldsm_x4(kbase + src, kf);
    ldsm_x4(vbase + src, vf);
#pragma unroll
    for (int e = 0; e < 4; ++e) xf[e] = gate_pair_x<kScaled>(kf[e], vf[e], s, mx);
    const int c = cg * 8 + rr;
    const uint32_t dst = (tg >> 3) * kKBlockBytes + c * kRowBytes + (((tg & 7) ^ rr) << 4);
    stsm_x4_trans(xbase + dst, xf);
  }
  return mx;
}

// Largest |k v| (float bits) over the 32 rows x 64 channels gate warp gw converts from the
// time-major, 128-byte-swizzled k and v tiles (the same fragments as the X build).  Once per
// sequence run.
__device__ __forceinline__ uint32_t kv_absmax(uint32_t kbase, uint32_t vbase, int gw, int lane) {
  const int mat = lane >> 3, rr = lane & 7;
  uint32_t m = 0;
#pragma unroll 1
  for (int it = 0; it < 8; ++it) {
    const int bw = it * 4 + mat;
    const int tg = gw * 4 + (bw >> 3), cg = bw & 7;
    const uint32_t src = (tg * 8 + rr) * kRowBytes + ((cg ^ rr) << 4);
    uint32_t kf[4], vf[4];
    ldsm_x4(kbase + src, kf);
    ldsm_x4(vbase + src, vf);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p0 = __uint_as_float(kf[e] << 16) * __uint_as_float(vf[e] << 16);
      const float p1 = __uint_as_float(kf[e] & 0xFFFF0000u) * __uint_as_float(vf[e] & 0xFFFF0000u);
      m = max(m, max(__float_as_uint(fabsf(p0)), __float_as_uint(fabsf(p1))));
    }
  }
  return __reduce_max_sync(0xffffffffu, m);
}

// Filter taps of the tile's kNG groups, staged once per sequence run by the 128 gate threads:
// group gg's taps start at hz + gg (258 + halo) + 2, and hz_g[i] = fp16(h[g kNG + gg][i - 127])
// for 0 <= i - 127 < l_h, else 0, for -2 <= i < 256 + halo.  One coalesced pass over the
// filters instead of each band lane fetching its own taps.  The loads (tap_load) are issued
// into registers and written to shared memory later (tap_store), so their latency can overlap
// other work.
template <int kPer>
__device__ __forceinline__ void tap_load(float (&v)[kPer], const float *hblk, int l_h, int halo,
                                         int ng, int tid) {
  const int stride = 258 + halo;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int e = tid + k * kGroupThreads;
    const int gg = e / stride, idx = e - gg * stride - 2 - 127;
    v[k] = (gg < ng && idx >= 0 && idx < l_h) ? __ldg(hblk + gg * l_h + idx) : 0.f;
  }
}

template <int kPer>
__device__ __forceinline__ void tap_store(uint16_t *hz, const float (&v)[kPer], int halo, int ng,
                                          int tid, bool &over) {
  const int n = ng * (258 + halo);
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int e = tid + k * kGroupThreads;
    if (e < n) {
      over |= fabsf(v[k]) > 65504.f;
      const __half hv = __float2half_rn(v[k]);
      hz[e] = *reinterpret_cast<const uint16_t *>(&hv);
    }
  }
}

// The same staging with group gg's taps scaled by 2^eh[gg] (exact) before the rounding to fp16.
template <int kNG, int kPer>
__device__ __forceinline__ void tap_store_scaled(uint16_t *hz, const float (&v)[kPer], int halo,
                                                 int tid, const int (&eh)[kNG]) {
  const int stride = 258 + halo, n = kNG * stride;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int e = tid + k * kGroupThreads;
    if (e < n) {
      const int gg = e / stride;
      float s = exp2i(eh[0]);
#pragma unroll
      for (int g2 = 1; g2 < kNG; ++g2)
        if (gg == g2) s = exp2i(eh[g2]);
      const __half hv = __float2half_rn(v[k] * s);
      hz[e] = *reinterpret_cast<const uint16_t *>(&hv);
    }
  }
}

// Largest |tap| of each of the tile's groups among this thread's staged taps, merged into
// hmax[gg] (float bits) with shared-memory atomics.
template <int kNG, int kPer>
__device__ __forceinline__ void tap_absmax(uint32_t *hmax, const float (&v)[kPer], int halo,
                                           int tid) {
  const int stride = 258 + halo;
  uint32_t m[kNG];
#pragma unroll
  for (int gg = 0; gg < kNG; ++gg) m[gg] = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int e = tid + k * kGroupThreads;
    const int gg = e / stride;
    const uint32_t a = __float_as_uint(fabsf(v[k]));
#pragma unroll
    for (int g2 = 0; g2 < kNG; ++g2)
      if (gg == g2) m[g2] = max(m[g2], a);
  }
#pragma unroll
  for (int gg = 0; gg < kNG; ++gg) {
    const uint32_t w = __reduce_max_sync(0xffffffffu, m[gg]);
    if ((tid & 31) == 0 && w) atomicMax(&hmax[gg], w);
  }
}

// The recomputation warp's work: y of one row of an out-of-range tile on the CUDA cores,
// y[t][c] = q[t][c] sum_j h[g(c)][j] k[t-j][c] v[t-j][c] for the 64 channels of block `blk`,
// taps in order, fp32, with the rows before the sequence from the history tensors (or zero),
// rounded to bf16 and written to y in global memory.  Eight channels at a time, through L2.
template <int kNG>
__device__ __forceinline__ void recompute_row_fp32(const Params &p, int blk, int b, long long t) {
  constexpr int kDG = kNC / kNG;
  if (t >= p.L) return;  // rows past the end do not exist
  const long long c0 = static_cast<long long>(blk) * kNC;
  const long long row = (static_cast<long long>(b) * p.L + t) * p.D + c0;
#pragma unroll 1
  for (int c8 = 0; c8 < kNC / 8; ++c8) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const float *hg = p.h + (static_cast<size_t>(blk) * kNG + (8 * c8) / kDG) * p.l_h;
#pragma unroll 1
    for (int j = 0; j < p.l_h; ++j) {
      const long long s = t - j;
      const __nv_bfloat16 *kr, *vr;
      if (s >= 0) {
        const long long off = (static_cast<long long>(b) * p.L + s) * p.D + c0;
        kr = p.k + off;
        vr = p.v + off;
      } else if (p.hist_tiles && p.Lh + s >= 0) {
        const long long off = (static_cast<long long>(b) * p.Lh + p.Lh + s) * p.D + c0;
        kr = p.kh + off;
        vr = p.vh + off;
      } else {
        break;
      }
      const uint4 kw = __ldg(reinterpret_cast<const uint4 *>(kr) + c8);
      const uint4 vw = __ldg(reinterpret_cast<const uint4 *>(vr) + c8);
      const float hj = __ldg(hg + j);
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, vv[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(kk[e] << 16) * __uint_as_float(vv[e] << 16);
        const float x1 = __uint_as_float(kk[e] & 0xFFFF0000u) * __uint_as_float(vv[e] & 0xFFFF0000u);
        acc[2 * e] = fmaf(hj, x0, acc[2 * e]);
        acc[2 * e + 1] = fmaf(hj, x1, acc[2 * e + 1]);
      }
    }
    const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(p.q + row) + c8);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    uint32_t ow[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xFFFF0000u);
      const __nv_bfloat162 yv = __floats2bfloat162_rn(q0 * acc[2 * e], q1 * acc[2 * e + 1]);
      ow[e] = *reinterpret_cast<const uint32_t *>(&yv);
    }
    reinterpret_cast<uint4 *>(p.y + row)[c8] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

// The Toeplitz band of one group in tensor memory.  Output rows are reversed (lane p holds
// time t0 + 127 - p) and K runs over input rows t0 - halo .. t0 + 127, so
//     A[p][kk] = h[127 + halo - p - kk]   (zero outside [0, l_h))  = hz_g[254 + halo - p - kk].
// Each of the 128 gate threads writes its own lane, 128 + halo K elements = band_cols columns
// (two fp16 K elements per 32-bit column, the lower K index in the low half), 32 (then 8)
// columns per tcgen05.st.  Column c needs hz_g[i0 - 2c] and hz_g[i0 - 2c - 1], i0 = 254 + halo
// - p: with i0 odd both lie in 32-bit word (i0 - 1) / 2 - c (halves swapped); with i0 even they
// are the low half of word i0 / 2 - c and the high half of the word below it.
template <int N>
__device__ __forceinline__ void band_chunk(uint32_t taddr, int c0, const uint32_t *hw, int m0,
                                           uint32_t sel) {
  uint32_t w[N + 1], r[N];
#pragma unroll
  for (int c = 0; c <= N; ++c) w[c] = hw[m0 - c0 - c];
#pragma unroll
  for (int c = 0; c < N; ++c) r[c] = __byte_perm(w[c], w[c + 1], sel);
  if constexpr (N == 32)
    tmem_st_32x32b_x32(taddr + c0, r);
  else
    tmem_st_32x32b_x8(taddr + c0, r);
}

__device__ __forceinline__ void build_band_tmem(uint32_t band_col, int band_cols,
                                                uint32_t tmem_base, const uint16_t *hzg, int halo,
                                                int quad, int lane) {
  const int row = quad * 32 + lane;
  const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + band_col;
  const int i0 = 254 + halo - row;
  const uint32_t sel = (i0 & 1) ? 0x1032u : 0x7610u;
  const uint32_t *hw = reinterpret_cast<const uint32_t *>(hzg);  // hzg is 4-byte aligned
  const int m0 = i0 >> 1;  // the lowest word read is m0 - band_cols >= -1 (the zero pad)
  int c0 = 0;
#pragma unroll 1
  for (; c0 + 32 <= band_cols; c0 += 32) band_chunk<32>(taddr, c0, hw, m0, sel);
#pragma unroll 1
  for (; c0 < band_cols; c0 += 8) band_chunk<8>(taddr, c0, hw, m0, sel);
  tmem_wait_st();
}

// kNG = 64 / d_g groups per tile (1, 2 or 4); MMA N = d_g.  kNH = ceil(halo / 128) earlier
// tiles feed each tile's product (1 for l_h <= 129, up to 5 for l_h <= 641).  kHooks builds
// the test instantiation: the waits between roles use p.wait_ns, and p.fault == 1 withholds
// the first accumulator arrive; the product instantiations carry neither.
template <int kNG, int kNH, bool kHooks = false>
__global__ void __launch_bounds__(kThreads, 1)
    fir_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_y,
                  const __grid_constant__ CUtensorMap tm_kh,
                  const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ Params p) {
  using Ly = Layout<kNH>;
  constexpr int kNQ = Ly::kNQ, kNX = Ly::kNX;
  constexpr int kOffKV = Ly::kOffKV, kOffQ = Ly::kOffQ, kOffX = Ly::kOffX, kOffBar = Ly::kOffBar,
                kOffMisc = Ly::kOffMisc;
  constexpr int kBarKVFull = Ly::kBarKVFull, kBarKVEmpty = Ly::kBarKVEmpty,
                kBarQFull = Ly::kBarQFull, kBarQEmpty = Ly::kBarQEmpty,
                kBarYReady = Ly::kBarYReady, kBarXFull = Ly::kBarXFull,
                kBarXEmpty = Ly::kBarXEmpty, kBarAccFull = Ly::kBarAccFull,
                kBarAccEmpty = Ly::kBarAccEmpty, kBarAFull = Ly::kBarAFull,
                kBarAEmpty = Ly::kBarAEmpty, kBarGate = Ly::kBarGate, kBarDone = Ly::kBarDone,
                kBarSegFull = Ly::kBarSegFull, kBarSegEmpty = Ly::kBarSegEmpty,
                kBarGateDone = Ly::kBarGateDone, kBarEpiDone = Ly::kBarEpiDone;
  constexpr int kNBad = Ly::kNBad;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *kv_st = smem + kOffKV;
  uint8_t *q_st = smem + kOffQ;
  uint8_t *x_st = smem + kOffX;
  uint16_t *hz = reinterpret_cast<uint16_t *>(smem + Ly::kOffHz);
  uint32_t *bad_count = reinterpret_cast<uint32_t *>(smem + Ly::kOffBad);
  long long *bad_w = reinterpret_cast<long long *>(smem + Ly::kOffBad + 8);
  uint32_t *segf = reinterpret_cast<uint32_t *>(smem + Ly::kOffSeg);
  uint32_t *maxw = reinterpret_cast<uint32_t *>(smem + Ly::kOffMax);  // [2][8]: |h| x4, |kv|
  const uint64_t lim = kHooks ? static_cast<uint64_t>(p.wait_ns) : kWaitTimeoutNs;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nwalk = p.paired ? gridDim.x / 2 : gridDim.x;
  const long long bx = p.paired ? blockIdx.x / 2 : blockIdx.x;
  const int gmul = p.paired ? 2 : 1, goff = p.paired ? static_cast<int>(blockIdx.x & 1) : 0;
  const long long per = p.W / nwalk, rem = p.W % nwalk;
  const long long w_begin = bx * per + (bx < rem ? bx : rem);
  const long long w_end = w_begin + per + (bx < rem ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < Ly::kNKV; ++i) {
      mbar_init(&bars[kBarKVFull + i], 1);
      mbar_init(&bars[kBarKVEmpty + i], kGroupThreads);
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(&bars[kBarQFull + i], 1);
      mbar_init(&bars[kBarQEmpty + i], 1);
      mbar_init(&bars[kBarYReady + i], kGroupThreads);
    }
    for (int i = 0; i < kNX; ++i) {
      mbar_init(&bars[kBarXFull + i], kGroupThreads);
      mbar_init(&bars[kBarXEmpty + i], 1);
    }
    for (int i = 0; i < kNAcc; ++i) {
      mbar_init(&bars[kBarAccFull + i], 1);
      mbar_init(&bars[kBarAccEmpty + i], kGroupThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarAFull + i], kGroupThreads);
      mbar_init(&bars[kBarAEmpty + i], 1);
    }
    mbar_init(&bars[kBarGate], kGroupThreads);
    mbar_init(&bars[kBarDone], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarSegFull + i], 1);   // gate warp 0, lane 0
      mbar_init(&bars[kBarSegEmpty + i], 4);  // lane 0 of each epilogue warp
    }
    mbar_init(&bars[kBarGateDone], 4);        // lane 0 of each gate warp
    mbar_init(&bars[kBarEpiDone], 1);         // the epilogue thread that issued the stores
    for (int i = 0; i < 16; ++i) maxw[i] = 0;
    *bad_count = 0;
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_y);
    if (p.hist_tiles) {
      tma_prefetch_desc(&tm_kh);
      tma_prefetch_desc(&tm_vh);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // Everything above touches no global memory, so under a programmatic dependent launch it
  // overlaps the end of the previous kernel.  From here on the inputs may be read.
  griddep_wait();
  griddep_launch_dependents();
  // Thread 0 is also the k/v producer: it queues the first k/v stages right away, before the
  // CTA-wide barrier (no other thread touches those stages yet).
  WorkIter kv_it(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
  // k and v of one item into stage `slot`: tiles i < 0 from the history tensors.
  auto load_kv = [&](uint32_t slot, const Item &t) {
    uint8_t *dst = kv_st + slot * 2 * kTileBytes;
    const bool h = t.i < 0;
    const int row = h ? p.Lh + t.i * kTM : t.i * kTM;
    tma_load_3d(dst, h ? &tm_kh : &tm_k, &bars[kBarKVFull + slot], t.g * kNC, row, t.b);
    tma_load_3d(dst + kTileBytes, h ? &tm_vh : &tm_v, &bars[kBarKVFull + slot], t.g * kNC, row,
                t.b);
  };
  Item kv_t;
  uint32_t kv_count = 0;
  bool kv_done = false;
  if (threadIdx.x == 0) {
    while (kv_count < Ly::kNKV) {
      if (!kv_it.next(kv_t)) {
        kv_done = true;
        break;
      }
      mbar_arrive_expect_tx(&bars[kBarKVFull + kv_count], 2 * kTileBytes);
      load_kv(kv_count, kv_t);
      ++kv_count;
    }
  }
  // The gate threads issue the loads of the first run's filter taps now; they land while the
  // CTA-wide barrier below completes and are written to shared memory after it.
  float taps[Ly::kPer];
  const bool gate_role = warp >= kWarpGate0 && warp < kWarpGate0 + 4;
  if (gate_role && w_begin < w_end) {
    const int g0 = static_cast<int>((w_begin / p.nT) / p.B) * gmul + goff;
    tap_load(taps, p.h + static_cast<size_t>(g0) * kNG * p.l_h, p.l_h, p.halo, kNG,
             threadIdx.x - kWarpGate0 * 32);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpTma) {
    // ---------------------------------------------------------------- TMA producer: k, v
    if (lane == 0) {
      uint32_t kc = kv_count;
      while (!kv_done && kv_it.next(kv_t)) {
        const Item &t = kv_t;
        const int ks = kc % Ly::kNKV;
        if (!thread_wait(&bars[kBarKVEmpty + ks], ((kc / Ly::kNKV) & 1) ^ 1, abort, lim)) break;
        mbar_arrive_expect_tx(&bars[kBarKVFull + ks], 2 * kTileBytes);
        load_kv(ks, t);
        ++kc;
      }
      // Every load this thread issued must land before the CTA may exit.
      for (uint32_t n = kc > Ly::kNKV ? kc - Ly::kNKV : 0; n < kc; ++n)
        drain_wait(&bars[kBarKVFull + n % Ly::kNKV], (n / Ly::kNKV) & 1);
    }
  } else if (warp == kWarpTmaQ) {
    // ---------------------------------------------------------------- TMA producer: q
    if (lane == 0) {
      WorkIter it(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
      Item t;
      uint32_t qc = 0;
      while (it.next(t)) {
        if (t.halo) continue;
        const int qs = qc % kNQ;
        if (!thread_wait(&bars[kBarQEmpty + qs], ((qc / kNQ) & 1) ^ 1, abort, lim)) break;
        mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes);
        tma_load_3d(q_st + qs * kTileBytes, &tm_q, &bars[kBarQFull + qs], t.g * kNC, t.i * kTM,
                    t.b);
        ++qc;
      }
      for (uint32_t n = qc > kNQ ? qc - kNQ : 0; n < qc; ++n)
        drain_wait(&bars[kBarQFull + n % kNQ], (n / kNQ) & 1);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      WorkIter it(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
      Item t;
      uint32_t xc = 0, ac = 0, seg_x0 = 0;
      int cur_seg = -1, x_seg = -1;
      constexpr int kDG = kNC / kNG;
      const uint32_t idesc = umma_idesc_f16_f32(kTM, kDG, 0);  // N = d_g, B K-major
      const int hsteps = p.halo / 16;
      // B = X^T, K-major with 128-byte swizzle: k-step s of a slot starts at K-block s / 4
      // (8 KB each) plus 32 bytes per step inside the 128-byte rows; group gg's rows start
      // gg * d_g channel rows (gg * d_g * 128 bytes) into the block.  Slot n starts n * 16 KB
      // after slot 0 (descriptor address field in 16-byte units).
      const uint64_t bd_x0 = umma_smem_desc(smem_u32(x_st), 16, 1024, 2);
      // History k-step j covers input rows t0 - halo + 16 j ..; counted from the start of the
      // oldest history tile (kNH tiles back) that is row hrow0 + 16 j.
      const int hrow0 = kNH * kTM - p.halo;
      while (it.next(t)) {
        const int xs = xc % kNX;
        if (t.seg != x_seg) {  // first item (halo or output) of a segment
          x_seg = t.seg;
          seg_x0 = xc;
        }
        if (!thread_wait(&bars[kBarXFull + xs], (xc / kNX) & 1, abort, lim)) break;
        if (t.halo) {
          ++xc;
          continue;
        }
        // band set of this segment and how often it was filled before (nbuf is 1 or 2)
        const int pa = p.nbuf == 2 ? (t.seg & 1) : 0;
        if (t.seg != cur_seg) {
          cur_seg = t.seg;
          const int use = p.nbuf == 2 ? (t.seg >> 1) : t.seg;
          if (!thread_wait(&bars[kBarAFull + pa], use & 1, abort, lim)) break;
        }
        const int as = ac % kNAcc;
        if (!thread_wait(&bars[kBarAccEmpty + as], ((ac / kNAcc) & 1) ^ 1, abort, lim)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kNC;
        const uint32_t band0 = tmem_base + kBandCol0 + pa * kNG * p.band_cols;
        // A (group gg's band) advances 8 columns (16 K elements) per k-step.  History steps
        // whose rows lie before the start of the sequence (and its history) are zero and skipped.
        const int jstart = max(0, (p.halo - (t.i + p.hist_tiles) * kTM) / 16);
        uint32_t a_run[kNG];  // next band column of each group
#pragma unroll
        for (int gg = 0; gg < kNG; ++gg) a_run[gg] = band0 + gg * p.band_cols + 8 * jstart;
        uint32_t acc = 0;     // 0 only for the first MMA of each group's chain
        for (int j = jstart; j < hsteps; ++j) {
          const int u = hrow0 + 16 * j;
          // with one history tile (u < 128) the slot is the same for every step
          const uint32_t slot = (xc + kNX - kNH + (kNH == 1 ? 0 : (u >> 7))) % kNX;
          const int st = (u & (kTM - 1)) >> 4;
          const uint64_t bdj = bd_x0 + (slot * (kTileBytes >> 4) + (st >> 2) * (kKBlockBytes >> 4) +
                                        (st & 3) * 2);
#pragma unroll
          for (int gg = 0; gg < kNG; ++gg) {
            umma_f16_ts(d_tmem + gg * kDG, a_run[gg], bdj + gg * (kDG * 8), idesc, acc);
            a_run[gg] += 8;
          }
          acc = 1;
        }
        {
          const uint64_t bd0 = bd_x0 + xs * (kTileBytes >> 4);
#pragma unroll
          for (int st = 0; st < kTM / 16; ++st) {
            const uint64_t bdj = bd0 + ((st >> 2) * (kKBlockBytes >> 4) + (st & 3) * 2);
#pragma unroll
            for (int gg = 0; gg < kNG; ++gg) {
              umma_f16_ts(d_tmem + gg * kDG, a_run[gg], bdj + gg * (kDG * 8), idesc, acc);
              a_run[gg] += 8;
            }
            acc = 1;
          }
        }
        // (test hook: withholding the first tile's arrive makes the epilogue's bounded wait
        // run out, which exercises the timeout path)
        if (!(kHooks && p.fault == 1 && ac == 0)) umma_commit(&bars[kBarAccFull + as]);
        // X slots go back to the gate warps after their last reader: the slot kNH items back
        // is read by no later tile; at the end of a segment every slot still held is free.
        if (xc >= seg_x0 + kNH) umma_commit(&bars[kBarXEmpty + (xc - kNH) % kNX]);
        if (t.last) {
          for (uint32_t n = xc + 1 > seg_x0 + kNH ? xc + 1 - kNH : seg_x0; n <= xc; ++n)
            umma_commit(&bars[kBarXEmpty + n % kNX]);
          umma_commit(&bars[kBarAEmpty + pa]);
        }
        ++xc;
        ++ac;
      }
      // Every MMA this thread issued must complete before TMEM is freed.
      umma_commit(&bars[kBarDone]);
      drain_wait(&bars[kBarDone], 0);
    }
  } else if (warp >= kWarpGate0 && warp < kWarpGate0 + 4) {
    // ---------------------------------------------------------------- pre-gate + band build
    WorkIter it(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
    Item t{};
    uint32_t kc = 0, xc = 0, gphase = 0;
    const int gtid = threadIdx.x - kWarpGate0 * 32, gw = warp - kWarpGate0;
    constexpr uint32_t kReadMask = ((2u << kNH) - 1u) | 0x80000000u;
    float sx = 1.f;        // 2^ex of the current run
    // This warp's range flags of its last items (bit 0 = the newest); bit 31 stays set for a
    // run whose scales were clamped (all its tiles go to fp32).
    uint32_t recent = 0;
    // One item (halo or output tile) of the current run: X^T into its slot, then the range
    // flags; an output tile reads its own rows and those of the kNH items before it.
    float first_mx = 0.f;  // this lane's largest scaled |x| of the run's first tile
    auto gate_item = [&](auto scaled, bool built) -> bool {
      constexpr bool kScaled = decltype(scaled)::value;
      const int ks = kc % Ly::kNKV, xs = xc % kNX;
      float mx = first_mx;  // the run's first tile was converted at the run's start
      if (!built) {
        if (!warp_wait(&bars[kBarKVFull + ks], (kc / Ly::kNKV) & 1, abort, lim)) return false;
        if (!warp_wait(&bars[kBarXEmpty + xs], ((xc / kNX) & 1) ^ 1, abort, lim)) return false;
        const uint32_t kbase = smem_u32(kv_st + ks * 2 * kTileBytes);
        mx = gate_x_tile<kScaled>(kbase, kbase + kTileBytes, smem_u32(x_st + xs * kTileBytes),
                                  gw, lane, sx);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarKVEmpty + ks]);
      mbar_arrive(&bars[kBarXFull + xs]);
      // an fp16 overflow, or every value of some lane tiny but not zero (fp16 subnormals, or
      // values that rounded to zero); the bits of a non-negative float order like the float
      const uint32_t mb = __float_as_uint(mx);
      const bool lane_bad = mb > kF16MaxBits || mb - 1u < kXTinyBits - 1u;
      recent = (recent << 1) | (__any_sync(0xffffffffu, lane_bad) ? 1u : 0u);
      if ((recent & kReadMask) && !t.halo && lane == 0) {
        // list the output tile for the recomputation warp
        const uint32_t n = atomicAdd(bad_count, 1u);
        if (n < kNBad) bad_w[n] = (static_cast<long long>(t.g / gmul) * p.B + t.b) * p.nT + t.i;
      }
      ++kc;
      ++xc;
      return true;
    };
    bool have = it.next(t), ok = true;
    while (have && ok) {
      // ------------------------------------ start of a sequence run (segment)
      const int seg = t.seg, par = seg & 1;
      ok = false;
      do {
        if (seg > 0) {
          // every gate thread has finished reading the previous taps ...
          tap_load(taps, p.h + static_cast<size_t>(t.g) * kNG * p.l_h, p.l_h, p.halo, kNG, gtid);
          mbar_arrive(&bars[kBarGate]);
          if (!warp_wait(&bars[kBarGate], gphase++ & 1, abort, lim)) break;
        }
        // ... the largest |h| of each group, once all have merged theirs ...
        tap_absmax<kNG>(maxw + 8 * par, taps, p.halo, gtid);
        mbar_arrive(&bars[kBarGate]);
        if (!warp_wait(&bars[kBarGate], gphase++ & 1, abort, lim)) break;
        int eh[kNG];
        bool run_bad = false;  // the run's scales were clamped: all its tiles go to fp32
#pragma unroll
        for (int gg = 0; gg < kNG; ++gg) eh[gg] = tap_scale_exp(maxw[8 * par + gg], run_bad);
        tap_store_scaled<kNG>(hz, taps, p.halo, gtid, eh);
        // ... and has written its share of the new ones
        mbar_arrive(&bars[kBarGate]);
        if (!warp_wait(&bars[kBarGate], gphase++ & 1, abort, lim)) break;
        const int pa = p.nbuf == 2 ? par : 0, use = p.nbuf == 2 ? (seg >> 1) : seg;
        if (use > 0 && !warp_wait(&bars[kBarAEmpty + pa], (use - 1) & 1, abort, lim)) break;
#pragma unroll 1
        for (int gg = 0; gg < kNG; ++gg)
          build_band_tmem(kBandCol0 + (pa * kNG + gg) * p.band_cols, p.band_cols, tmem_base,
                          hz + gg * (258 + p.halo) + 2, p.halo, warp & 3, lane);
        tc_fence_before_sync();
        mbar_arrive(&bars[kBarAFull + pa]);
        // x's scale from the largest |k v| of the run's first tile: that tile is converted
        // unscaled first (no scale is the usual case), every warp merges its maximum, and the
        // tile is converted again, scaled, only if the run needs it
        const int ks = kc % Ly::kNKV, xs = xc % kNX;
        if (!warp_wait(&bars[kBarKVFull + ks], (kc / Ly::kNKV) & 1, abort, lim)) break;
        if (!warp_wait(&bars[kBarXEmpty + xs], ((xc / kNX) & 1) ^ 1, abort, lim)) break;
        const uint32_t kbase = smem_u32(kv_st + ks * 2 * kTileBytes);
        const uint32_t xbase = smem_u32(x_st + xs * kTileBytes);
        const float m0 = gate_x_tile<false>(kbase, kbase + kTileBytes, xbase, gw, lane, 1.f);
        const uint32_t xm = __reduce_max_sync(0xffffffffu, __float_as_uint(m0));
        if (lane == 0 && xm) atomicMax(&maxw[8 * par + 4], xm);
        mbar_arrive(&bars[kBarGate]);
        if (!warp_wait(&bars[kBarGate], gphase++ & 1, abort, lim)) break;
        const int ex = x_scale_exp(maxw[8 * par + 4], eh[0], run_bad);
        if (ex != 0) gate_x_tile<true>(kbase, kbase + kTileBytes, xbase, gw, lane, exp2i(ex));
        first_mx = m0 * exp2i(ex);  // exact: the lane's maximum after the scale
        sx = exp2i(ex);
        uint32_t fexp = 0;
#pragma unroll
        for (int gg = 0; gg < kNG; ++gg)
          fexp |= (static_cast<uint32_t>(eh[gg] + ex) & 0xFFu) << (8 * gg);
        // the other parity's maxima were last read before this run's barriers: reset them
        if (gtid < 8) maxw[8 * (par ^ 1) + gtid] = 0;
        // hand the run's scale to the epilogue (its slot was last read for the run two back)
        if (gw == 0) {
          if (!warp_wait(&bars[kBarSegEmpty + par], ((seg >> 1) & 1) ^ 1, abort, lim)) break;
          if (lane == 0) {
            segf[par] = fexp;
            mbar_arrive(&bars[kBarSegFull + par]);
          }
        }
        recent = run_bad ? 0x80000000u : 0u;
        ok = true;
      } while (false);
      if (!ok) break;
      // ------------------------------------ the run's items, with or without x's scale (the
      // first one's X is built; it finishes like the others)
      bool first = true;
      if (sx == 1.f) {
        do {
          if (!(ok = gate_item(std::false_type(), first))) break;
          first = false;
          have = it.next(t);
        } while (have && t.seg == seg);
      } else {
        do {
          if (!(ok = gate_item(std::true_type(), first))) break;
          first = false;
          have = it.next(t);
        } while (have && t.seg == seg);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarGateDone]);
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ---------------------------------------------------------------- epilogue
    const int et = threadIdx.x - kWarpEpi0 * 32;
    const int quad = warp & 3;               // TMEM lanes this warp may read
    const int row_lane = quad * 32 + lane;   // MMA row = TMEM lane
    const int r = kTM - 1 - row_lane;        // tile row (time offset) of that lane
    WorkIter it(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
    Item t{};
    uint32_t ac = 0, qc = 0;
    // One output tile: the accumulator (divided by the run's 2^(eh + ex) when kScaled), times q,
    // rounded to bf16 over the q stage, and stored.
    auto epi_item = [&](auto scaled, uint32_t rfexp) -> bool {
      constexpr bool kScaled = decltype(scaled)::value;
      const int as = ac % kNAcc, qs = qc % kNQ;
      if (!warp_wait(&bars[kBarAccFull + as], (ac / kNAcc) & 1, abort, lim)) return false;
      tc_fence_after_sync();
      uint32_t a0[32], a1[32];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + as * kNC;
      tmem_ld_32x32b_x32(taddr, a0);
      tmem_ld_32x32b_x32(taddr + 32, a1);
      tmem_wait_ld();
      reg_fence(a0);
      reg_fence(a1);
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarAccEmpty + as]);
      if (kScaled) {
        // group gg's accumulator carries 2^(eh[gg] + ex) (byte gg of rfexp): divided out exactly
        constexpr int kDG = kNC / kNG;
        float fs[kNG];
#pragma unroll
        for (int gg = 0; gg < kNG; ++gg)
          fs[gg] = exp2i(-static_cast<int>(static_cast<int8_t>(rfexp >> (8 * gg))));
#pragma unroll
        for (int ch = 0; ch < 32; ++ch) {
          a0[ch] = __float_as_uint(__uint_as_float(a0[ch]) * fs[ch / kDG]);
          a1[ch] = __float_as_uint(__uint_as_float(a1[ch]) * fs[(ch + 32) / kDG]);
        }
      }
      if (!warp_wait(&bars[kBarQFull + qs], (qc / kNQ) & 1, abort, lim)) return false;
      uint8_t *qrow = q_st + qs * kTileBytes + r * (kNC * 2);
#pragma unroll kEpiUnroll
      for (int c = 0; c < 8; ++c) {
        uint4 *ptr = reinterpret_cast<uint4 *>(qrow + ((c ^ (r & 7)) << 4));
        const uint4 qv = *ptr;
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ch = 8 * c + 2 * e;
          const float acc0 = __uint_as_float(ch < 32 ? a0[ch] : a1[ch - 32]);
          const float acc1 = __uint_as_float(ch + 1 < 32 ? a0[ch + 1] : a1[ch + 1 - 32]);
          const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xFFFF0000u);
          const __nv_bfloat162 yv = __floats2bfloat162_rn(q0 * acc0, q1 * acc1);
          ow[e] = *reinterpret_cast<const uint32_t *>(&yv);
        }
        *ptr = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarYReady + qs]);
      bool sok = true;
      if (et == 0) {
        sok = thread_wait(&bars[kBarYReady + qs], (qc / kNQ) & 1, abort, lim);
        if (sok) {
          tma_store_3d(&tm_y, q_st + qs * kTileBytes, t.g * kNC, t.i * kTM, t.b);
          bulk_commit_group();
          // One store stays in flight: once the previous tile's store has read its shared
          // memory, that q/y stage goes back to the producer.
          bulk_wait_group_read<1>();
          if (qc > 0) mbar_arrive(&bars[kBarQEmpty + (qc + kNQ - 1) % kNQ]);
        }
      }
      if (!__all_sync(0xffffffffu, sok)) return false;
      ++ac;
      ++qc;
      return true;
    };
    bool have = it.next(t), ok = true;
    while (have && ok) {
      // the run's scale exponents (eh + ex per group), once per run
      const int seg = t.seg, sp = seg & 1;
      if (!warp_wait(&bars[kBarSegFull + sp], (seg >> 1) & 1, abort, lim)) break;
      const uint32_t rfexp = segf[sp];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarSegEmpty + sp]);
      if (rfexp == 0) {
        do {
          if (!t.halo && !(ok = epi_item(std::false_type(), 0u))) break;
          have = it.next(t);
        } while (have && t.seg == seg);
      } else {
        do {
          if (!t.halo && !(ok = epi_item(std::true_type(), rfexp))) break;
          have = it.next(t);
        } while (have && t.seg == seg);
      }
    }
    if (et == 0) {
      // The stores must have read their shared memory before the CTA exits; their global
      // writes complete with the grid.
      bulk_wait_group_read<0>();
      if (qc > 0) mbar_arrive(&bars[kBarQEmpty + (qc + kNQ - 1) % kNQ]);
      // Where the gate listed tiles for recomputation, their rows are rewritten after this
      // CTA's stores have landed.
      if (thread_wait(&bars[kBarGateDone], 0, abort, lim) &&
          *reinterpret_cast<volatile uint32_t *>(bad_count) > 0) {
        bulk_wait_group<0>();
        fence_proxy_async_global();
      }
      mbar_arrive(&bars[kBarEpiDone]);
    }
  } else if (warp == kWarpFix) {
    // ---------------------------------------------------------------- recomputation
    // Once the gate has listed every tile (it finishes well before the epilogue) there is
    // usually nothing to do and the warp leaves.  Otherwise it sleeps until the epilogue is done
    // (possibly most of the kernel, so with a long limit) and recomputes the listed tiles in
    // fp32: 4 rows of each per lane.
    // Both waits sleep between polls: this warp shares its scheduler with a gate warp and an
    // epilogue warp, and spinning would take issue slots from them.
    auto sleep_wait = [&](int bar) -> bool {
      const uint64_t t0 = global_timer_ns();
      for (;;) {
        if (mbar_try_wait(smem_u32(&bars[bar]), 0)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > kFixWaitNs) {
          *abort = 1;
          atomicOr(&g_device_status, kTimeoutBit);
          return false;
        }
        __nanosleep(1000);
      }
    };
    const bool go = sleep_wait(kBarGateDone) &&
                    *reinterpret_cast<volatile uint32_t *>(bad_count) > 0 &&
                    sleep_wait(kBarEpiDone);
    const uint32_t nbad = go ? *reinterpret_cast<volatile uint32_t *>(bad_count) : 0u;
    if (nbad > 0) {
      if (nbad <= static_cast<uint32_t>(kNBad)) {
        for (uint32_t k = 0; k < nbad; ++k) {
          const long long w = bad_w[k], seq = w / p.nT;
          const int i = static_cast<int>(w - seq * p.nT);
          const int g = static_cast<int>(seq / p.B) * gmul + goff;
          const int b = static_cast<int>(seq % p.B);
          for (int rr = lane; rr < kTM; rr += 32)
            recompute_row_fp32<kNG>(p, g, b, static_cast<long long>(i) * kTM + rr);
        }
      } else {  // more than the list holds: every output tile of this CTA
        WorkIter all(w_begin, w_end, p.nT, p.B, gmul, goff, kNH, p.hist_tiles);
        Item t;
        while (all.next(t))
          if (!t.halo)
            for (int rr = lane; rr < kTM; rr += 32)
              recompute_row_fp32<kNG>(p, t.g, t.b, static_cast<long long>(t.i) * kTM + rr);
      }
      if (lane == 0) atomicOr(&g_device_status, kF16RangeBit);
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace tc
}  // namespace hyena
