// fir_tc_bwd.cuh -- tcgen05 kernel of the backward of the gated grouped causal FIR (bf16,
// d_g = 64): the anti-causal product and the filter gradient.
//
// For y = q * z, z = h_g conv x, x = k * v and the upstream gradient dy (page "04.
// Hardware-aware convolution kernels", Sec. 7 backward; Sec. 2-3 block-Toeplitz form):
//   dq = dy * z                      -- the forward kernel with dy in the place of q (host)
//   dk = dx * v,  dv = dx * k        dx = T^T (q * dy)  (anti-causal: the transposed product)
//   dh[g][j] = sum_{t, c in g} dz[t, c] x[t - j, c],  dz = q * dy
// This kernel reads q, k, v, dy once and writes dk, dv once; dh leaves as one fp32 partial per
// (CTA, segment), summed in a fixed order by fir_bwd_tc_reduce_kernel (the two passes of Sec. 7).
// Computing dq here as well (recomputing z = T x on chip) saves three tensor streams but puts
// 40 MMAs on every 128 x 64 tile; with 24 this kernel and the forward each run near the HBM
// bound, which measured faster than the fused form.
//
// Tiles are 128 time rows x 64 channels (one group).  Each CTA walks contiguous tile ranges
// like the forward kernel, but every sequence run ("segment", tiles lo..hi) in DECREASING time,
// so the anti-causal product of a tile finds the next tile's dz already on chip.
//
// B200 specifics:
//  * The forward's Toeplitz band in tensor memory, A[p][kk] = h[127 + halo - p - kk], computes
//    z = T x with output lane p = time t0 + 127 - p.  Fed with dz in REVERSED time (operand row
//    kk = time t0 + 127 + halo - kk), the same band yields lane p = dx[t0 + p]: dz tiles are
//    stored time-reversed, and the anti-causal chain is the causal chain with the next tile in
//    the place of the previous one.  The band is built from the filter taps staged in shared
//    memory, as in the forward.
//  * dh as a GEMM: C[m][n] = sum_c x[t0 + m, c] dz[tau(n), c] over the 256 dz times of tiles
//    i and i+1 (two M128 N128 K64 MMAs with both operands MN-major, read straight from the
//    channel-major fp16 tiles).  C accumulates in tensor memory over a whole segment; the lag
//    j = tau(n) - t0 - m is constant along anti-diagonals, which the epilogue sums once per
//    segment.
//  * Tensor memory (512 columns): two dx accumulators [0, 128) (the MMA issuer fills one while
//    the epilogue drains the other), band [128, 256), C [256, 512).
//  * Warp roles as the forward: 0 TMA k/v, 10 TMA q/dy (fetching into L2 ahead of the loads
//    as well measured slower: prefetched tiles were evicted before use), 1 MMA issuer + TMEM owner, 2-5 operand build
//    (x = k v; dz = q dy written over the q tile; the band), 6-9 epilogue.  The epilogue copies
//    its k, v rows from the stage into registers, releases it, and stores dk, dv rows directly;
//    it also sums the dh anti-diagonals.  Every wait is bounded; a timeout raises
//    HYENA_DEVICE_TIMEOUT and all roles drain and leave.
//  * Operand range.  x, dz and h are rounded to fp16 unscaled.  Where a value of any of them
//    lies above 65504 (it would round to inf), or a group's taps all lie below 2^-10 (deep in
//    fp16's subnormals), the gate writes the call's token into the range flag in the host's
//    workspace and raises HYENA_DEVICE_F16_RANGE; the host queues the fp32 CUDA-core backward
//    behind this kernel, gated on that token, and it rewrites dk, dv and dh.  (Scaling x and dz
//    by powers of two chosen per CTA, as the forward does per sequence run, measured 233 us
//    instead of 192 us at the MR shape: this kernel's time follows its gate and epilogue
//    warps' critical path, and every added step on it showed in the total.)
#pragma once
#include "fir_tc.cuh"

namespace hyena {
namespace tcb {

using tc::kTM;
using tc::kNC;
using tc::kTileBytes;
using tc::kKBlockBytes;
using tc::kRowBytes;
using tc::kGroupThreads;
using tc::kTimeoutBit;
using tc::kF16RangeBit;
constexpr int kMaxHalo = 128;  // one tile of history: l_h - 1 <= 128

constexpr int kNKV = 3;   // k/v stages (32 KB each)
constexpr int kNQ = 3;    // q stages; each becomes the tile's fp16 dz (channel-major, reversed)
constexpr int kNDY = 2;   // dy stages (free once dz is built)
constexpr int kNX = 2;    // fp16 x tiles, channel-major (free once the tile's dh product ran)

constexpr uint32_t kColDX = 0, kColBand = 128, kColC = 256;
constexpr int kTmemCols = 512;

constexpr int kRedLd = 17;                       // 32 x 16 scratch per epilogue warp, padded
constexpr int kPartLen = 132;                    // dh taps per epilogue warp (l_h <= 129)
constexpr int kHzStride = 258 + kMaxHalo;        // staged fp16 taps of one group (see tc::tap_load)
constexpr int kTapPer = (kHzStride + kGroupThreads - 1) / kGroupThreads;

constexpr int kOffKV = 0;
constexpr int kOffQ = kOffKV + kNKV * 2 * kTileBytes;
constexpr int kOffDY = kOffQ + kNQ * kTileBytes;
constexpr int kOffX = kOffDY + kNDY * kTileBytes;
constexpr int kOffRed = kOffX + kNX * kTileBytes;
constexpr int kOffPart = kOffRed + 4 * 32 * kRedLd * 4;
constexpr int kOffHz = kOffPart + 4 * kPartLen * 4;
constexpr int kOffBar = (kOffHz + kHzStride * 2 + 15) / 16 * 16;

constexpr int kBarKVFull = 0;
constexpr int kBarKVEmpty = kBarKVFull + kNKV;
constexpr int kBarQFull = kBarKVEmpty + kNKV;
constexpr int kBarQEmpty = kBarQFull + kNQ;
constexpr int kBarDYFull = kBarQEmpty + kNQ;
constexpr int kBarDYEmpty = kBarDYFull + kNDY;
constexpr int kBarXFull = kBarDYEmpty + kNDY;
constexpr int kBarXEmpty = kBarXFull + kNX;
constexpr int kBarDZFull = kBarXEmpty + kNX;   // dz built over q stage s
constexpr int kBarGateRead = kBarDZFull + kNQ; // every gate thread has read its q, dy fragments
constexpr int kBarGate = kBarGateRead + 1;     // the gate threads among themselves (tap staging)
constexpr int kBarDXFull = kBarGate + 1;       // two of each: one per accumulator set
constexpr int kBarDXEmpty = kBarDXFull + 2;
constexpr int kBarCFull = kBarDXEmpty + 2;
constexpr int kBarCEmpty = kBarCFull + 1;
constexpr int kBarAFull = kBarCEmpty + 1;
constexpr int kBarAEmpty = kBarAFull + 1;
constexpr int kBarRedDone = kBarAEmpty + 1;
constexpr int kBarDone = kBarRedDone + 1;
constexpr int kNumBars = kBarDone + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
// kOffMisc: TMEM address, abort flag, then each gate warp's largest |h| of the segment (float
// bits; two sets by segment parity)
constexpr int kMiscTapMax = 8;
constexpr int kSmemBytes = kOffMisc + 48 + 1024;  // + slack for 1024-byte alignment
// A group whose largest |tap| is below 2^-10 (float bits): its taps sit in fp16's subnormals.
constexpr uint32_t kTapTinyBits = 0x3A800000u;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget of one CTA exceeded");

constexpr int kThreads = 352;
constexpr int kWarpTmaKV = 0, kWarpMma = 1, kWarpGate0 = 2, kWarpEpi0 = 6, kWarpTmaQ = 10;

struct Params {
  const float *h;     // [G, l_h]
  float *partial;     // [gridDim.x * max_segs, l_h]: dh of each (CTA, segment)
  int *seg_group;     // [gridDim.x * max_segs]: the group of each partial
  int *seg_count;     // [gridDim.x]: segments each CTA wrote
  int B, L, l_h;
  int G;              // groups = 64-channel blocks = D / 64
  int halo;           // multiple of 16, >= l_h - 1, <= 128
  int band_cols;      // (128 + halo) / 2
  int nT;             // tiles per sequence
  long long W;        // tiles of the walk: G * B * nT
  int max_segs;       // partial slots per CTA
  long long D;        // channels (row length of every [B, L, D] tensor)
  __nv_bfloat16 *dk, *dv;  // outputs, written by rows
  unsigned *range_flag;    // set to range_token where an operand leaves fp16's range
  unsigned range_token;    // this call's token (the host's fallback kernels run on a match)
};

enum ItemKind { kNextHalo = 0, kMain = 1 };

// One unit of a CTA's walk.  A segment (tiles lo..hi of one (group, batch) sequence) is walked
//   [next-halo: tile hi + 1's q, dy -> dz only]  main hi, main hi-1, ..., main lo.
struct BItem {
  int kind;
  int g, b, i;        // group, sequence, tile (next-halo: tile hi + 1)
  int lo, hi, seg;
  bool seg_first;     // first item of its segment
};

struct BwdWalk {
  long long w, w_end;
  int nT, B, seg, state, g, b, lo, hi, i;
  __device__ BwdWalk(long long w_begin, long long w_end_, int nT_, int B_)
      : w(w_begin), w_end(w_end_), nT(nT_), B(B_), seg(-1), state(0), g(0), b(0), lo(0), hi(0),
        i(0) {}
  __device__ bool next(BItem &it) {
    bool first = false;
    if (state == 0) {
      if (w >= w_end) return false;
      const long long seq = w / nT;
      lo = static_cast<int>(w - seq * nT);
      const long long left = w_end - w;
      const int n = static_cast<int>(left < nT - lo ? left : nT - lo);
      hi = lo + n - 1;
      g = static_cast<int>(seq / B);
      b = static_cast<int>(seq - static_cast<long long>(g) * B);
      w += n;
      ++seg;
      i = hi;
      state = hi + 1 < nT ? 1 : 2;
      first = true;
    }
    it.g = g;
    it.b = b;
    it.lo = lo;
    it.hi = hi;
    it.seg = seg;
    it.seg_first = first;
    if (state == 1) {
      it.kind = kNextHalo;
      it.i = hi + 1;
      state = 2;
    } else {
      it.kind = kMain;
      it.i = i;
      if (i == lo)
        state = 0;
      else
        --i;
    }
    return true;
  }
};

// fp16 channel-major tile (the operand layout of fir_tc_kernel's x) from two time-major bf16
// tiles a, b of one stage: out = fp16(a * b).  kRev stores time reversed (position m holds time
// 127 - m): the ldmatrix rows of each 8-time block are taken in reverse order, so the transposed
// store writes the block's times high to low, into block 15 - tg.
template <bool kRev>
__device__ __forceinline__ void gate_tile(uint32_t abase, uint32_t bbase, uint32_t obase,
                                          int gw, int lane, bool &over) {
  const int mat = lane >> 3, rr = lane & 7;
  const int srow = kRev ? 7 - rr : rr;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bw = it * 4 + mat;
    const int tg = gw * 4 + (bw >> 3), cg = bw & 7;
    const uint32_t src = (tg * 8 + srow) * kRowBytes + ((cg ^ srow) << 4);
    uint32_t af[4], bf[4], of[4];
    ldsm_x4(abase + src, af);
    ldsm_x4(bbase + src, bf);
#pragma unroll
    for (int e = 0; e < 4; ++e) of[e] = tc::gate_pair(af[e], bf[e], over);
    const int c = cg * 8 + rr;
    const int tgo = kRev ? 15 - tg : tg;
    const uint32_t dst = (tgo >> 3) * kKBlockBytes + c * kRowBytes + (((tgo & 7) ^ rr) << 4);
    stsm_x4_trans(obase + dst, of);
  }
}

// dz = fp16(q * dy), time-reversed and channel-major (gate_tile<true>'s layout), written over
// the q tile itself: every gate thread reads its fragments of both tiles first, the group meets
// at `read_bar` (no thread overwrites q before all have read it), then the transposed blocks
// are stored.  False if the wait gave up.
__device__ __forceinline__ bool gate_dz_inplace(uint32_t qbase, uint32_t dybase, int gw, int lane,
                                                bool &over, uint64_t *read_bar, uint32_t parity,
                                                volatile int *abort) {
  const int mat = lane >> 3, rr = lane & 7, srow = 7 - rr;
  uint32_t dz[8][4];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bw = it * 4 + mat;
    const int tg = gw * 4 + (bw >> 3), cg = bw & 7;
    const uint32_t src = (tg * 8 + srow) * kRowBytes + ((cg ^ srow) << 4);
    uint32_t af[4], bf[4];
    ldsm_x4(qbase + src, af);
    ldsm_x4(dybase + src, bf);
#pragma unroll
    for (int e = 0; e < 4; ++e) dz[it][e] = tc::gate_pair(af[e], bf[e], over);
  }
  mbar_arrive(read_bar);
  if (!tc::warp_wait(read_bar, parity, abort)) return false;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int bw = it * 4 + mat;
    const int tg = gw * 4 + (bw >> 3), cg = bw & 7;
    const int c = cg * 8 + rr, tgo = 15 - tg;
    const uint32_t dst = (tgo >> 3) * kKBlockBytes + c * kRowBytes + (((tgo & 7) ^ rr) << 4);
    stsm_x4_trans(qbase + dst, dz[it]);
  }
  return true;
}

// The Toeplitz chain of one 128-row tile (the forward's MMA sequence for one group): band
// columns from `band0`, 8 per K16 step; K covers the halo rows of `hist` (positions
// 128 - halo .. 127), or zeros when hist < 0, then the 128 rows of `cur`.
__device__ __forceinline__ void toeplitz_chain(uint32_t d_tmem, uint32_t band0, uint32_t x_st,
                                               int hist, int cur, int halo, uint32_t idesc) {
  const int hsteps = halo / 16;
  uint32_t a = band0, acc = 0;
  if (hist >= 0) {
    const uint64_t bd0 = umma_smem_desc(x_st + hist * kTileBytes, 16, 1024, 2);
    const int s0 = (kTM - halo) / 16;
    for (int j = 0; j < hsteps; ++j) {
      const int st = s0 + j;
      umma_f16_ts(d_tmem, a, bd0 + ((st >> 2) * (kKBlockBytes >> 4) + (st & 3) * 2), idesc, acc);
      a += 8;
      acc = 1;
    }
  } else {
    a += 8 * hsteps;
  }
  const uint64_t bd0 = umma_smem_desc(x_st + cur * kTileBytes, 16, 1024, 2);
#pragma unroll
  for (int st = 0; st < kTM / 16; ++st) {
    umma_f16_ts(d_tmem, a, bd0 + ((st >> 2) * (kKBlockBytes >> 4) + (st & 3) * 2), idesc, acc);
    a += 8;
    acc = 1;
  }
}

// C[:, n0 .. n0 + 127] (+)= X^T-tile (M = 128 times, K = 64 channels) x dz-tile (N = 128
// positions): 4 K16 steps over channel rows, both operands MN-major with 128-byte swizzle
// (64-element atoms 8 KB apart, 8-channel groups 1 KB apart).
__device__ __forceinline__ void c_chain(uint32_t d_tmem, uint32_t a_tile, uint32_t b_tile,
                                        uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint64_t ad = umma_smem_desc(a_tile + s * 2048, kKBlockBytes, 1024, 2);
    const uint64_t bd = umma_smem_desc(b_tile + s * 2048, kKBlockBytes, 1024, 2);
    umma_f16(d_tmem, ad, bd, idesc, (accumulate || s > 0) ? 1u : 0u);
  }
}

// Rows of a 64-channel tile in shared memory (128-byte rows, 16-byte chunks swizzled by the row).
__device__ __forceinline__ uint4 *row_chunk(uint8_t *tile, int r, int c) {
  return reinterpret_cast<uint4 *>(tile + r * kRowBytes + ((c ^ (r & 7)) << 4));
}

// One 16-byte shared-memory load that the compiler may neither repeat nor move: a stage's
// rows must be read before the stage is handed back to its producer, and a plain load could be
// re-issued after that point (rematerialised instead of spilled) and see the next tile.
// An instruction that reads every loaded register, so the warp waits until the loads have
// returned their data (an empty asm would emit nothing and wait for nothing).
__device__ __forceinline__ void consume_rows(const uint4 (&r)[8]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    asm volatile("{\n\t.reg .b32 t;\n\txor.b32 t, %0, %1;\n\txor.b32 t, t, %2;\n\t"
                 "xor.b32 t, t, %3;\n\t}" ::"r"(r[c].x), "r"(r[c].y), "r"(r[c].z), "r"(r[c].w));
}

__device__ __forceinline__ uint4 lds_v4(const void *p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_u32(p))
               : "memory");
  return r;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float (&o)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = __uint_as_float(w[e] << 16);
    o[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t *>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}


__global__ void __launch_bounds__(kThreads, 1)
    fir_tc_bwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_dy, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *kv_st = smem + kOffKV;
  uint8_t *q_st = smem + kOffQ;
  uint8_t *dy_st = smem + kOffDY;
  uint8_t *x_st = smem + kOffX;
  float *red = reinterpret_cast<float *>(smem + kOffRed);
  float *part = reinterpret_cast<float *>(smem + kOffPart);
  uint16_t *hz = reinterpret_cast<uint16_t *>(smem + kOffHz);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  uint32_t *tapmax = reinterpret_cast<uint32_t *>(smem + kOffMisc + kMiscTapMax);  // [2][4]
  volatile int *abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nct = gridDim.x, bx = blockIdx.x;
  const long long per = p.W / nct, rem = p.W % nct;
  const long long w_begin = bx * per + (bx < rem ? bx : rem);
  const long long w_end = w_begin + per + (bx < rem ? 1 : 0);

  if (threadIdx.x == 0) {
    // k/v stages are released by both readers: the operand builders and the epilogue
    for (int i = 0; i < kNKV; ++i) {
      mbar_init(&bars[kBarKVFull + i], 1);
      mbar_init(&bars[kBarKVEmpty + i], 2 * kGroupThreads);
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(&bars[kBarQFull + i], 1);
      mbar_init(&bars[kBarQEmpty + i], 1);  // released by the MMA once dz is used up
      mbar_init(&bars[kBarDZFull + i], kGroupThreads);
    }
    for (int i = 0; i < kNDY; ++i) {
      mbar_init(&bars[kBarDYFull + i], 1);
      mbar_init(&bars[kBarDYEmpty + i], kGroupThreads);
    }
    for (int i = 0; i < kNX; ++i) {
      mbar_init(&bars[kBarXFull + i], kGroupThreads);
      mbar_init(&bars[kBarXEmpty + i], 1);
    }
    mbar_init(&bars[kBarGateRead], kGroupThreads);
    mbar_init(&bars[kBarGate], kGroupThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarDXFull + i], 1);
      mbar_init(&bars[kBarDXEmpty + i], kGroupThreads);
    }
    mbar_init(&bars[kBarCFull], 1);
    mbar_init(&bars[kBarCEmpty], kGroupThreads);
    mbar_init(&bars[kBarAFull], kGroupThreads);
    mbar_init(&bars[kBarAEmpty], 1);
    mbar_init(&bars[kBarRedDone], kGroupThreads);
    mbar_init(&bars[kBarDone], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // Launched with programmatic stream serialisation after the dq forward, which only starts
  // its dependents once it has itself waited for every earlier kernel of the stream: the
  // inputs are complete when this grid starts, and nothing here reads what the forward writes
  // (dq), so the work overlaps the forward's last tiles without a grid-dependency wait.
  griddep_launch_dependents();
  // The gate threads issue the loads of the first segment's filter taps before the barrier
  // (and each gate warp leaves the group's largest |h| among its taps in tapmax[0][warp]).
  bool over = false;
  float taps[kTapPer];
  auto tap_share_max = [&](uint32_t *slot) {
    uint32_t hm = 0;
#pragma unroll
    for (int k2 = 0; k2 < kTapPer; ++k2) hm = max(hm, __float_as_uint(fabsf(taps[k2])));
    hm = __reduce_max_sync(0xffffffffu, hm);
    if (lane == 0) *slot = hm;
  };
  if (warp >= kWarpGate0 && warp < kWarpGate0 + 4 && w_begin < w_end) {
    const int g0 = static_cast<int>((w_begin / p.nT) / p.B);
    tc::tap_load(taps, p.h + static_cast<size_t>(g0) * p.l_h, p.l_h, p.halo, 1,
                 threadIdx.x - kWarpGate0 * 32);
    tap_share_max(&tapmax[warp - kWarpGate0]);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpTmaKV) {
    // ------------------------------------------------------------ TMA producer: k, v
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      BwdWalk it(w_begin, w_end, p.nT, p.B);
      BItem t;
      uint32_t kc = 0;
      while (it.next(t)) {
        if (t.kind != kMain) continue;
        const int ks = kc % kNKV;
        if (!tc::thread_wait(&bars[kBarKVEmpty + ks], ((kc / kNKV) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(&bars[kBarKVFull + ks], 2 * kTileBytes);
        uint8_t *dst = kv_st + ks * 2 * kTileBytes;
        tma_load_3d(dst, &tm_k, &bars[kBarKVFull + ks], t.g * kNC, t.i * kTM, t.b);
        tma_load_3d(dst + kTileBytes, &tm_v, &bars[kBarKVFull + ks], t.g * kNC, t.i * kTM, t.b);
        ++kc;
      }
      for (uint32_t n = kc > kNKV ? kc - kNKV : 0; n < kc; ++n)
        tc::drain_wait(&bars[kBarKVFull + n % kNKV], (n / kNKV) & 1);
    }
  } else if (warp == kWarpTmaQ) {
    // ------------------------------------------------------------ TMA producer: q, dy
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_dy);
      BwdWalk it(w_begin, w_end, p.nT, p.B);
      BItem t;
      uint32_t qc = 0, dc = 0;
      while (it.next(t)) {
        const int qs = qc % kNQ, ds = dc % kNDY;
        if (!tc::thread_wait(&bars[kBarQEmpty + qs], ((qc / kNQ) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes);
        tma_load_3d(q_st + qs * kTileBytes, &tm_q, &bars[kBarQFull + qs], t.g * kNC, t.i * kTM,
                    t.b);
        ++qc;
        if (!tc::thread_wait(&bars[kBarDYEmpty + ds], ((dc / kNDY) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(&bars[kBarDYFull + ds], kTileBytes);
        tma_load_3d(dy_st + ds * kTileBytes, &tm_dy, &bars[kBarDYFull + ds], t.g * kNC,
                    t.i * kTM, t.b);
        ++dc;
      }
      for (uint32_t n = qc > kNQ ? qc - kNQ : 0; n < qc; ++n)
        tc::drain_wait(&bars[kBarQFull + n % kNQ], (n / kNQ) & 1);
      for (uint32_t n = dc > kNDY ? dc - kNDY : 0; n < dc; ++n)
        tc::drain_wait(&bars[kBarDYFull + n % kNDY], (n / kNDY) & 1);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      BwdWalk it(w_begin, w_end, p.nT, p.B);
      BItem t;
      uint32_t xc = 0, dzc = 0, dxc = 0, cc = 0;
      const uint32_t id_t = umma_idesc_f16_f32(kTM, kNC, 0);        // Toeplitz chains
      const uint32_t id_c = umma_idesc_f16_f32_mn(kTM, 128, 1, 1);  // dh products
      const uint32_t band0 = tmem_base + kColBand;
      const uint32_t xs_base = smem_u32(x_st), dz_base = smem_u32(q_st);  // dz over q
      bool lo_init = false, hi_init = false;
      while (it.next(t)) {
        if (t.kind == kNextHalo) {
          if (!tc::thread_wait(&bars[kBarDZFull + dzc % kNQ], (dzc / kNQ) & 1, abort)) break;
          ++dzc;
          continue;
        }
        if (t.i == t.hi) {  // first main tile: this segment's band
          if (!tc::thread_wait(&bars[kBarAFull], t.seg & 1, abort)) break;
        }
        const int xs = xc % kNX, ds = dzc % kNQ;
        if (!tc::thread_wait(&bars[kBarXFull + xs], (xc / kNX) & 1, abort)) break;
        if (!tc::thread_wait(&bars[kBarDZFull + ds], (dzc / kNQ) & 1, abort)) break;
        const bool has_next = t.i + 1 < p.nT;
        const int dn = (dzc + kNQ - 1) % kNQ;  // dz of tile i + 1 (previous acquisition)
        // dx(i): the band against dz of tiles i+1 (halo rows) and i
        const int xb = dxc & 1;
        if (!tc::thread_wait(&bars[kBarDXEmpty + xb], ((dxc >> 1) & 1) ^ 1, abort)) break;
        tc_fence_after_sync();
        toeplitz_chain(tmem_base + kColDX + 64 * xb, band0, dz_base, has_next ? dn : -1, ds,
                       p.halo, id_t);
        umma_commit(&bars[kBarDXFull + xb]);
        ++dxc;
        // C += x(i) dz(i), x(i) dz(i+1)
        if (t.i == t.hi) {
          if (!tc::thread_wait(&bars[kBarCEmpty], (cc & 1) ^ 1, abort)) break;
          tc_fence_after_sync();
          lo_init = hi_init = false;
        }
        c_chain(tmem_base + kColC, xs_base + xs * kTileBytes, dz_base + ds * kTileBytes, id_c,
                lo_init);
        lo_init = true;
        if (has_next) {
          c_chain(tmem_base + kColC + 128, xs_base + xs * kTileBytes, dz_base + dn * kTileBytes,
                  id_c, hi_init);
          hi_init = true;
          umma_commit(&bars[kBarQEmpty + dn]);  // dz(i+1) is used up
        }
        umma_commit(&bars[kBarXEmpty + xs]);    // x(i) is used up
        if (t.i == t.lo) {
          umma_commit(&bars[kBarQEmpty + ds]);  // dz(lo) is used up
          umma_commit(&bars[kBarCFull]);
          umma_commit(&bars[kBarAEmpty]);
          ++cc;
        }
        ++xc;
        ++dzc;
      }
      // Every MMA this thread issued must complete before TMEM is freed.
      umma_commit(&bars[kBarDone]);
      tc::drain_wait(&bars[kBarDone], 0);
    }
  } else if (warp >= kWarpGate0 && warp < kWarpGate0 + 4) {
    // ------------------------------------------------------------ operand build
    BwdWalk it(w_begin, w_end, p.nT, p.B);
    BItem t;
    uint32_t kc = 0, qc = 0, dc = 0, xc = 0, rc = 0, gphase = 0;
    const int gw = warp - kWarpGate0, gtid = threadIdx.x - kWarpGate0 * 32;
    while (it.next(t)) {
      if (t.seg_first) {
        const uint32_t *tm = tapmax + 4 * (t.seg & 1);
        if (t.seg > 0) {
          if (!tc::warp_wait(&bars[kBarAEmpty], (t.seg - 1) & 1, abort)) break;
          tc::tap_load(taps, p.h + static_cast<size_t>(t.g) * p.l_h, p.l_h, p.halo, 1, gtid);
          tap_share_max(&tapmax[4 * (t.seg & 1) + gw]);
          // every gate thread has finished reading the previous taps (and left its warp's
          // largest tap) ...
          mbar_arrive(&bars[kBarGate]);
          if (!tc::warp_wait(&bars[kBarGate], gphase++ & 1, abort)) break;
        }
        // (segment 0's maxima were left before the CTA barrier; a slot set is rewritten two
        // segments later, after a barrier that every reader of it has passed)
        const uint32_t hmax = max(max(tm[0], tm[1]), max(tm[2], tm[3]));
        over |= hmax != 0 && hmax < kTapTinyBits;
        tc::tap_store(hz, taps, p.halo, 1, gtid, over);
        // ... and has written its share of the new ones
        mbar_arrive(&bars[kBarGate]);
        if (!tc::warp_wait(&bars[kBarGate], gphase++ & 1, abort)) break;
        tc::build_band_tmem(kColBand, p.band_cols, tmem_base, hz + 2, p.halo, warp & 3, lane);
        tc_fence_before_sync();
        mbar_arrive(&bars[kBarAFull]);
      }
      const bool need_x = t.kind == kMain;
      const int ks = kc % kNKV, qs = qc % kNQ, ds = dc % kNDY, xs = xc % kNX;
      if (need_x) {
        if (!tc::warp_wait(&bars[kBarKVFull + ks], (kc / kNKV) & 1, abort)) break;
        if (!tc::warp_wait(&bars[kBarXEmpty + xs], ((xc / kNX) & 1) ^ 1, abort)) break;
        const uint32_t kb = smem_u32(kv_st + ks * 2 * kTileBytes);
        gate_tile<false>(kb, kb + kTileBytes, smem_u32(x_st + xs * kTileBytes), gw, lane, over);
      }
      if (!tc::warp_wait(&bars[kBarQFull + qs], (qc / kNQ) & 1, abort)) break;
      if (!tc::warp_wait(&bars[kBarDYFull + ds], (dc / kNDY) & 1, abort)) break;
      if (!gate_dz_inplace(smem_u32(q_st + qs * kTileBytes), smem_u32(dy_st + ds * kTileBytes),
                           gw, lane, over, &bars[kBarGateRead], rc & 1, abort))
        break;
      ++rc;
      fence_proxy_async_smem();
      if (need_x) {
        mbar_arrive(&bars[kBarXFull + xs]);
        mbar_arrive(&bars[kBarKVEmpty + ks]);  // the epilogue is the stage's other reader
        ++kc;
        ++xc;
      }
      mbar_arrive(&bars[kBarDZFull + qs]);
      mbar_arrive(&bars[kBarDYEmpty + ds]);
      ++qc;
      ++dc;
    }
    if (over) {  // (per thread: a lane's own products; writers all store the same token)
      atomicOr(&g_device_status, kF16RangeBit);
      *p.range_flag = p.range_token;
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    // Thread = one tile row.  It copies its k, v rows from the input stage into registers and
    // releases the stage at once; dk, dv rows go straight out with streaming stores.
    const int et = threadIdx.x - kWarpEpi0 * 32;
    const int quad = warp & 3;              // TMEM lanes this warp may read
    const int row_lane = quad * 32 + lane;  // MMA row = TMEM lane
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    float *rbuf = red + quad * 32 * kRedLd;
    float *pw = part + quad * kPartLen;
    BwdWalk it(w_begin, w_end, p.nT, p.B);
    BItem t;
    uint32_t dxc = 0, cc = 0, kc = 0;
    int nseg = 0;
    while (it.next(t)) {
      if (t.kind != kMain) continue;
      // dk = dx * v and dv = dx * k (dx lane p = time 128 i + p)
      const int ks = kc % kNKV;
      const uint32_t kcount = kc++;
      const long long tt = static_cast<long long>(t.i) * kTM + row_lane;
      if (!tc::warp_wait(&bars[kBarKVFull + ks], (kcount / kNKV) & 1, abort)) break;
      uint4 kr[8], vr[8];
      uint8_t *ktile = kv_st + ks * 2 * kTileBytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        kr[c] = lds_v4(row_chunk(ktile, row_lane, c));
        vr[c] = lds_v4(row_chunk(ktile + kTileBytes, row_lane, c));
      }
      const int xb = dxc & 1;
      if (!tc::warp_wait(&bars[kBarDXFull + xb], (dxc >> 1) & 1, abort)) break;
      tc_fence_after_sync();
      uint32_t a0[32], a1[32];
      tmem_ld_32x32b_x32(tl + kColDX + 64 * xb, a0);
      tmem_ld_32x32b_x32(tl + kColDX + 64 * xb + 32, a1);
      tmem_wait_ld();
      reg_fence(a0);
      reg_fence(a1);
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarDXEmpty + xb]);
      ++dxc;
      if (tt < p.L) {
        const long long off = (static_cast<long long>(t.b) * p.L + tt) * p.D +
                              static_cast<long long>(t.g) * kNC;
        uint4 *dk = reinterpret_cast<uint4 *>(p.dk + off);
        uint4 *dv = reinterpret_cast<uint4 *>(p.dv + off);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float kf[8], vf[8], ok8[8], ov8[8];
          unpack_bf16x8(kr[c], kf);
          unpack_bf16x8(vr[c], vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = 8 * c + e;
            const float dx = __uint_as_float(ch < 32 ? a0[ch] : a1[ch - 32]);
            ok8[e] = dx * vf[e];
            ov8[e] = dx * kf[e];
          }
          __stcs(dk + c, pack_bf16x8(ok8));
          __stcs(dv + c, pack_bf16x8(ov8));
        }
      }
      // The stage goes back to the producer (whose next TMA write to it is an async-proxy
      // access) only once every row load has returned its data and is ordered before the
      // arrive: an arrive issued right after the loads let the next tile's TMA write land under
      // them (seen as sporadic wrong rows in one warp's quarter of a tile).
      consume_rows(kr);
      consume_rows(vr);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarKVEmpty + ks]);
      if (t.i != t.lo) continue;
      // end of the segment: the dh sums
      if (!tc::warp_wait(&bars[kBarCFull], cc & 1, abort)) break;
      tc_fence_after_sync();
      for (int j = lane; j < kPartLen; j += 32) pw[j] = 0.f;
      __syncwarp();
      const bool hi_valid = (t.hi + 1 < p.nT) || (t.hi > t.lo);
      // C[m][n]: lag j = J0 - d with d = (m - 32 quad) + (n - n0), along anti-diagonals
      for (int n0 = 0; n0 < (hi_valid ? 256 : 128); n0 += 16) {
        const int J0 = (n0 < 128 ? 127 : 383) - n0 - 32 * quad;
        if (J0 < 0 || J0 - 46 >= p.l_h) continue;
        uint32_t v[16];
        tmem_ld_32x32b_x16(tl + kColC + n0, v);
        tmem_wait_ld();
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) rbuf[lane * kRedLd + i2] = __uint_as_float(v[i2]);
        __syncwarp();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int d = lane + 32 * h2;
          if (d <= 46) {
            float s = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < 16; ++k2) {
              const int pl = d - k2;
              if (pl >= 0 && pl < 32) s += rbuf[pl * kRedLd + k2];
            }
            const int j = J0 - d;
            if (j >= 0 && j < p.l_h) pw[j] += s;
          }
        }
        __syncwarp();
      }
      mbar_arrive(&bars[kBarRedDone]);
      if (!tc::warp_wait(&bars[kBarRedDone], cc & 1, abort)) break;
      if (nseg < p.max_segs) {  // the host sizes max_segs for every walk; never false
        const long long slot = static_cast<long long>(blockIdx.x) * p.max_segs + nseg;
        for (int j = et; j < p.l_h; j += kGroupThreads)
          p.partial[slot * p.l_h + j] = part[j] + part[kPartLen + j] + part[2 * kPartLen + j] +
                                        part[3 * kPartLen + j];
        if (et == 0) p.seg_group[slot] = t.g;
      }
      // released only after every thread has read `part`: the next segment's sums reuse it
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarCEmpty]);
      ++cc;
      ++nseg;
    }
    if (et == 0) p.seg_count[blockIdx.x] = nseg < p.max_segs ? nseg : p.max_segs;
  }

  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// dh[g][j] = sum over the CTAs whose tile range meets group g's tiles (in CTA order) and their
// segments (in order) of the partials of group g.  CTA c owns walk positions
// [c per + min(c, rem), ...) of the W tiles ordered (group, batch, time); group g owns
// [g span, (g + 1) span) with span = B nT.
__device__ __forceinline__ long long cta_of(long long w, long long per, long long rem) {
  const long long big = rem * (per + 1);
  return w < big ? w / (per + 1) : rem + (w - big) / per;
}

__global__ void __launch_bounds__(256)
    fir_bwd_tc_reduce_kernel(const float *__restrict__ partial, const int *__restrict__ seg_group,
                             const int *__restrict__ seg_count, int max_segs,
                             float *__restrict__ dh, int G, int l_h, long long per, long long rem,
                             long long span) {
  griddep_wait();  // launched with programmatic stream serialisation after fir_tc_bwd_kernel
  const long long n = static_cast<long long>(G) * l_h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(e / l_h), j = static_cast<int>(e % l_h);
    const long long c0 = cta_of(g * span, per, rem), c1 = cta_of((g + 1) * span - 1, per, rem);
    float s = 0.f;
    for (long long c = c0; c <= c1; ++c) {
      const int ns = seg_count[c];
      for (int k = 0; k < ns; ++k) {
        const long long slot = c * max_segs + k;
        if (seg_group[slot] == g) s += partial[slot * l_h + j];
      }
    }
    dh[e] = s;
  }
}

}  // namespace tcb
}  // namespace hyena
