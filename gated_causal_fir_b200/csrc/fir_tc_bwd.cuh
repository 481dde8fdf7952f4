// fir_tc_bwd.cuh -- fused tcgen05 backward of the gated grouped causal FIR (bf16, d_g = 64).
//
// For y = q * z, z = h_g conv x, x = k * v and the upstream gradient dy (page "04.
// Hardware-aware convolution kernels", Sec. 7 backward; Sec. 2-3 block-Toeplitz form):
//   dq = dy * z                      z  = T x           (causal Toeplitz product)
//   dk = dx * v,  dv = dx * k        dx = T^T (q * dy)  (anti-causal: the transposed product)
//   dh[g][j] = sum_{t, c in g} dz[t, c] x[t - j, c],  dz = q * dy
// One kernel reads q, k, v, dy once and writes dq, dk, dv once; dh leaves as one fp32 partial
// per (CTA, segment), summed in a fixed order by fir_bwd_tc_reduce_kernel.
//
// Tiles are 128 time rows x 64 channels (one group).  Each CTA walks contiguous tile ranges
// like the forward kernel, but every sequence run ("segment", tiles lo..hi) in DECREASING time,
// so the anti-causal product of a tile finds the next tile's dz already on chip.  The causal
// product of tile i+1 is issued once tile i's x exists (one tile of lag), which costs one extra
// dy stage instead of keeping k and v longer.
//
// B200 specifics:
//  * One Toeplitz band in tensor memory serves both products.  The forward's band
//    A[p][kk] = h[127 + halo - p - kk] multiplies x rows t0 - halo + kk into output lane
//    p = time t0 + 127 - p.  Fed with dz in REVERSED time (operand row kk = time
//    t0 + 127 + halo - kk), the same band yields lane p = dx[t0 + p]: so dz tiles are stored
//    time-reversed, and the anti-causal chain is the causal chain's code with the next tile in
//    the place of the previous one.
//  * dh as a GEMM: C[m][n] = sum_c x[t0 + m, c] dz[tau(n), c] over the 256 dz times of tiles
//    i and i+1 (two M128 N128 K64 MMAs with both operands MN-major, read straight from the
//    channel-major fp16 tiles the Toeplitz chains use).  C accumulates in tensor memory over a
//    whole segment; the lag j = tau(n) - t0 - m is constant along anti-diagonals, which the
//    epilogue sums once per segment.
//  * Tensor memory (512 columns): z accumulator [0, 64), dx accumulator [64, 128), band
//    [128, 128 + band_cols), C [256, 512).
//  * Warp roles as the forward: 0 TMA k/v, 10 TMA q/dy (both fetch their tiles into L2 a few
//    items ahead, then into shared memory), 1 MMA issuer + TMEM owner, 2-5 operand build
//    (x = k v; dz = q dy written over the q tile; the band), 6-9 epilogue.  The epilogue reads
//    its k, v, dy rows from global memory (L2-resident: just loaded) and stores dq, dk, dv rows
//    directly, so every input stage is released as soon as its operand is built; it also sums
//    the dh anti-diagonals.  Every wait is bounded; a timeout raises HYENA_DEVICE_TIMEOUT and
//    all roles drain and leave.
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

// The Toeplitz band of one group in tensor memory, each lane fetching its own taps from
// global memory.  Output rows are reversed (lane p holds
// time t0 + 127 - p) and K runs over input rows t0 - halo .. t0 + 127, so
//     A[p][kk] = h[127 + halo - p - kk]   (zero outside [0, l_h)),  rounded to fp16.
// Each of the 128 gate threads writes its own lane: 128 + halo K elements = band_cols columns.
// Columns [c0, c0 + N) of one lane's band row: 2 N taps loaded together, then one store.
template <int N>
__device__ __forceinline__ void band_chunk_gmem(uint32_t taddr, int c0, int row, const float *hg,
                                           int l_h, int halo, bool &over) {
  uint32_t r[N];
#pragma unroll
  for (int c = 0; c < N; ++c) {
    const int idx = kTM - 1 + halo - row - 2 * (c0 + c);  // tap of K element 2 (c0 + c)
    const float v0 = (idx >= 0 && idx < l_h) ? __ldg(hg + idx) : 0.f;
    const float v1 = (idx - 1 >= 0 && idx - 1 < l_h) ? __ldg(hg + idx - 1) : 0.f;
    over |= (fabsf(v0) > 65504.f) | (fabsf(v1) > 65504.f);
    const __half2 hv = __floats2half2_rn(v0, v1);
    r[c] = *reinterpret_cast<const uint32_t *>(&hv);
  }
  if constexpr (N == 32)
    tmem_st_32x32b_x32(taddr + c0, r);
  else
    tmem_st_32x32b_x8(taddr + c0, r);
}

__device__ __forceinline__ void build_band_gmem(uint32_t band_col, int band_cols,
                                                uint32_t tmem_base, const float *hg, int l_h,
                                                int halo, int quad, int lane, bool &over) {
  const int row = quad * 32 + lane;
  const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + band_col;
  int c0 = 0;
  // 32 columns (64 taps in flight) per step, then the 8-column remainder.
#pragma unroll 1
  for (; c0 + 32 <= band_cols; c0 += 32) band_chunk_gmem<32>(taddr, c0, row, hg, l_h, halo, over);
#pragma unroll 1
  for (; c0 < band_cols; c0 += 8) band_chunk_gmem<8>(taddr, c0, row, hg, l_h, halo, over);
  tmem_wait_st();
}


constexpr int kNKV = 2;   // k/v stages (32 KB each)
constexpr int kNQ = 3;    // q stages; each becomes the tile's fp16 dz (channel-major, reversed)
constexpr int kNDY = 3;   // dy stages
constexpr int kNX = 3;    // fp16 x tiles, channel-major
constexpr int kPrefetch = 3;  // items a producer fetches into L2 ahead of its loads

constexpr uint32_t kColZ = 0, kColDX = 64, kColBand = 128, kColC = 256;
constexpr int kTmemCols = 512;

constexpr int kRedLd = 17;                       // 32 x 16 scratch per epilogue warp, padded
constexpr int kPartLen = 132;                    // dh taps per epilogue warp (l_h <= 129)

constexpr int kOffKV = 0;
constexpr int kOffQ = kOffKV + kNKV * 2 * kTileBytes;
constexpr int kOffDY = kOffQ + kNQ * kTileBytes;
constexpr int kOffX = kOffDY + kNDY * kTileBytes;
constexpr int kOffRed = kOffX + kNX * kTileBytes;
constexpr int kOffPart = kOffRed + 4 * 32 * kRedLd * 4;
constexpr int kOffBar = kOffPart + 4 * kPartLen * 4;

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
constexpr int kBarZFull = kBarGateRead + 1;
constexpr int kBarZEmpty = kBarZFull + 1;
constexpr int kBarDXFull = kBarZEmpty + 1;
constexpr int kBarDXEmpty = kBarDXFull + 1;
constexpr int kBarCFull = kBarDXEmpty + 1;
constexpr int kBarCEmpty = kBarCFull + 1;
constexpr int kBarAFull = kBarCEmpty + 1;
constexpr int kBarAEmpty = kBarAFull + 1;
constexpr int kBarRedDone = kBarAEmpty + 1;
constexpr int kBarDone = kBarRedDone + 1;
constexpr int kNumBars = kBarDone + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
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
  const __nv_bfloat16 *k, *v, *dy;  // inputs the epilogue reads by rows
  __nv_bfloat16 *dq, *dk, *dv;      // outputs, written by rows
};

enum ItemKind { kNextHalo = 0, kMain = 1, kTail = 2 };

// One unit of a CTA's walk.  A segment (tiles lo..hi of one (group, batch) sequence) is walked
//   [next-halo: tile hi + 1's q, dy -> dz only]  main hi, main hi-1, ..., main lo,
//   tail: tile lo - 1's k, v -> x only (when lo > 0), then z of tile lo.
struct BItem {
  int kind;
  int g, b, i;        // group, sequence, tile (main: the tile; halos: the halo tile)
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
    } else if (state == 2) {
      it.kind = kMain;
      it.i = i;
      if (i == lo)
        state = 3;
      else
        --i;
    } else {
      it.kind = kTail;
      it.i = lo - 1;
      state = 0;
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
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nct = gridDim.x, bx = blockIdx.x;
  const long long per = p.W / nct, rem = p.W % nct;
  const long long w_begin = bx * per + (bx < rem ? bx : rem);
  const long long w_end = w_begin + per + (bx < rem ? 1 : 0);

  if (threadIdx.x == 0) {
    // k/v and dy stages are released by both readers: the operand builders and the epilogue
    // (the builders arrive twice for halo tiles, which the epilogue never reads)
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
      mbar_init(&bars[kBarDYEmpty + i], 2 * kGroupThreads);
    }
    for (int i = 0; i < kNX; ++i) {
      mbar_init(&bars[kBarXFull + i], kGroupThreads);
      mbar_init(&bars[kBarXEmpty + i], 1);
    }
    mbar_init(&bars[kBarGateRead], kGroupThreads);
    mbar_init(&bars[kBarZFull], 1);
    mbar_init(&bars[kBarZEmpty], kGroupThreads);
    mbar_init(&bars[kBarDXFull], 1);
    mbar_init(&bars[kBarDXEmpty], kGroupThreads);
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
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpTmaKV) {
    // ------------------------------------------------------------ TMA producer: k, v
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      BwdWalk it(w_begin, w_end, p.nT, p.B), pf(w_begin, w_end, p.nT, p.B);
      BItem t, u;
      auto kv_item = [](const BItem &x) { return x.kind == kMain || (x.kind == kTail && x.lo > 0); };
      // L2 prefetch runs kPrefetch loads ahead: the loads then find their tiles in L2.
      auto prefetch_next = [&]() {
        while (pf.next(u)) {
          if (!kv_item(u)) continue;
          tma_prefetch_l2_3d(&tm_k, u.g * kNC, u.i * kTM, u.b);
          tma_prefetch_l2_3d(&tm_v, u.g * kNC, u.i * kTM, u.b);
          return;
        }
      };
      for (int n = 0; n < kPrefetch; ++n) prefetch_next();
      uint32_t kc = 0;
      while (it.next(t)) {
        if (!kv_item(t)) continue;
        prefetch_next();
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
      BwdWalk it(w_begin, w_end, p.nT, p.B), pf(w_begin, w_end, p.nT, p.B);
      BItem t, u;
      auto prefetch_next = [&]() {
        while (pf.next(u)) {
          if (u.kind == kTail) continue;
          tma_prefetch_l2_3d(&tm_q, u.g * kNC, u.i * kTM, u.b);
          tma_prefetch_l2_3d(&tm_dy, u.g * kNC, u.i * kTM, u.b);
          return;
        }
      };
      for (int n = 0; n < kPrefetch; ++n) prefetch_next();
      uint32_t qc = 0, dc = 0;
      while (it.next(t)) {
        if (t.kind == kTail) continue;
        prefetch_next();
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
      uint32_t xc = 0, dzc = 0, zc = 0, dxc = 0, cc = 0;
      const uint32_t id_t = umma_idesc_f16_f32(kTM, kNC, 0);        // Toeplitz chains
      const uint32_t id_c = umma_idesc_f16_f32_mn(kTM, 128, 1, 1);  // dh products
      const uint32_t band0 = tmem_base + kColBand;
      const uint32_t xs_base = smem_u32(x_st), dz_base = smem_u32(q_st);  // dz over q
      bool lo_init = false, hi_init = false;
      bool ok = true;
      while (ok && it.next(t)) {
        if (t.kind == kNextHalo) {
          ok = tc::thread_wait(&bars[kBarDZFull + dzc % kNQ], (dzc / kNQ) & 1, abort);
          ++dzc;
          continue;
        }
        if (t.kind == kMain) {
          if (t.i == t.hi) {  // first main tile: this segment's band
            if (!tc::thread_wait(&bars[kBarAFull], t.seg & 1, abort)) break;
          }
          const int xs = xc % kNX, ds = dzc % kNQ;
          if (!tc::thread_wait(&bars[kBarXFull + xs], (xc / kNX) & 1, abort)) break;
          if (!tc::thread_wait(&bars[kBarDZFull + ds], (dzc / kNQ) & 1, abort)) break;
          const bool has_next = t.i + 1 < p.nT;
          const int dn = (dzc + kNQ - 1) % kNQ;  // dz of tile i + 1 (previous acquisition)
          // dx(i): the band against dz of tiles i+1 (halo rows) and i
          if (!tc::thread_wait(&bars[kBarDXEmpty], (dxc & 1) ^ 1, abort)) break;
          tc_fence_after_sync();
          toeplitz_chain(tmem_base + kColDX, band0, dz_base, has_next ? dn : -1, ds, p.halo,
                         id_t);
          umma_commit(&bars[kBarDXFull]);
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
            c_chain(tmem_base + kColC + 128, xs_base + xs * kTileBytes,
                    dz_base + dn * kTileBytes, id_c, hi_init);
            hi_init = true;
            umma_commit(&bars[kBarQEmpty + dn]);
          }
          // z(i+1): the band against x of tiles i (halo rows) and i+1
          if (t.i < t.hi) {
            const int xn = (xc + kNX - 1) % kNX;
            if (!tc::thread_wait(&bars[kBarZEmpty], (zc & 1) ^ 1, abort)) break;
            tc_fence_after_sync();
            toeplitz_chain(tmem_base + kColZ, band0, xs_base, xs, xn, p.halo, id_t);
            umma_commit(&bars[kBarZFull]);
            ++zc;
            umma_commit(&bars[kBarXEmpty + xn]);
          }
          if (t.i == t.lo) {
            umma_commit(&bars[kBarCFull]);
            ++cc;
          }
          ++xc;
          ++dzc;
          continue;
        }
        // tail: z(lo) against x of tile lo - 1 (when it exists) and lo
        const bool has_prev = t.lo > 0;
        const int xl = (xc + kNX - 1) % kNX, xp = xc % kNX;
        if (has_prev && !tc::thread_wait(&bars[kBarXFull + xp], (xc / kNX) & 1, abort)) break;
        if (!tc::thread_wait(&bars[kBarZEmpty], (zc & 1) ^ 1, abort)) break;
        tc_fence_after_sync();
        toeplitz_chain(tmem_base + kColZ, band0, xs_base, has_prev ? xp : -1, xl, p.halo, id_t);
        umma_commit(&bars[kBarZFull]);
        ++zc;
        umma_commit(&bars[kBarXEmpty + xl]);
        if (has_prev) {
          umma_commit(&bars[kBarXEmpty + xp]);
          ++xc;
        }
        umma_commit(&bars[kBarQEmpty + (dzc + kNQ - 1) % kNQ]);
        umma_commit(&bars[kBarAEmpty]);
      }
      // Every MMA this thread issued must complete before TMEM is freed.
      umma_commit(&bars[kBarDone]);
      tc::drain_wait(&bars[kBarDone], 0);
    }
  } else if (warp >= kWarpGate0 && warp < kWarpGate0 + 4) {
    // ------------------------------------------------------------ operand build
    BwdWalk it(w_begin, w_end, p.nT, p.B);
    BItem t;
    uint32_t kc = 0, qc = 0, dc = 0, xc = 0, rc = 0;
    const int gw = warp - kWarpGate0;
    bool over = false;
    while (it.next(t)) {
      if (t.seg_first) {
        if (t.seg > 0 && !tc::warp_wait(&bars[kBarAEmpty], (t.seg - 1) & 1, abort)) break;
        build_band_gmem(kColBand, p.band_cols, tmem_base, p.h + static_cast<size_t>(t.g) * p.l_h,
                            p.l_h, p.halo, warp & 3, lane, over);
        tc_fence_before_sync();
        mbar_arrive(&bars[kBarAFull]);
      }
      if (t.kind == kTail && t.lo == 0) continue;
      const bool need_x = t.kind != kNextHalo, need_dz = t.kind != kTail;
      const int ks = kc % kNKV, qs = qc % kNQ, ds = dc % kNDY, xs = xc % kNX;
      if (need_x) {
        if (!tc::warp_wait(&bars[kBarKVFull + ks], (kc / kNKV) & 1, abort)) break;
        if (!tc::warp_wait(&bars[kBarXEmpty + xs], ((xc / kNX) & 1) ^ 1, abort)) break;
        const uint32_t kb = smem_u32(kv_st + ks * 2 * kTileBytes);
        gate_tile<false>(kb, kb + kTileBytes, smem_u32(x_st + xs * kTileBytes), gw, lane, over);
      }
      if (need_dz) {
        if (!tc::warp_wait(&bars[kBarQFull + qs], (qc / kNQ) & 1, abort)) break;
        if (!tc::warp_wait(&bars[kBarDYFull + ds], (dc / kNDY) & 1, abort)) break;
        if (!gate_dz_inplace(smem_u32(q_st + qs * kTileBytes), smem_u32(dy_st + ds * kTileBytes),
                             gw, lane, over, &bars[kBarGateRead], rc & 1, abort))
          break;
        ++rc;
      }
      fence_proxy_async_smem();
      // this group is done with k, v (and dy); halo tiles have no second reader
      if (need_x) {
        mbar_arrive(&bars[kBarXFull + xs]);
        mbar_arrive_cnt(&bars[kBarKVEmpty + ks], t.kind == kTail ? 2 : 1);
        ++kc;
        ++xc;
      }
      if (need_dz) {
        mbar_arrive(&bars[kBarDZFull + qs]);
        mbar_arrive_cnt(&bars[kBarDYEmpty + ds], t.kind == kNextHalo ? 2 : 1);
        ++qc;
        ++dc;
      }
    }
    if (over) atomicOr(&g_device_status, kF16RangeBit);
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    // ------------------------------------------------------------ epilogue
    // Thread = one tile row.  It copies its k, v (and later dy) rows from the input stages into
    // registers and releases the stage at once; dq, dk, dv rows go straight out with streaming
    // stores, so no stage waits for an output to drain.
    const int et = threadIdx.x - kWarpEpi0 * 32;
    const int quad = warp & 3;              // TMEM lanes this warp may read
    const int row_lane = quad * 32 + lane;  // MMA row = TMEM lane
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    float *rbuf = red + quad * 32 * kRedLd;
    float *pw = part + quad * kPartLen;
    BwdWalk it(w_begin, w_end, p.nT, p.B);
    BItem t;
    uint32_t zc = 0, dxc = 0, cc = 0, kc = 0, dc = 0;
    int prev_ds = 0;        // dy stage of the previous main tile (its dq comes one step later)
    uint32_t prev_dc = 0;   // and that stage's use count
    int nseg = 0;
    // Element offset of row `tt` of sequence b, group g (channel 64 g), or -1 past the end.
    auto row_off = [&](int b, long long tt, int g) -> long long {
      return tt < p.L ? (static_cast<long long>(b) * p.L + tt) * p.D + static_cast<long long>(g) * kNC
                      : -1;
    };
    auto smem_row = [&](uint8_t *tile, int r, uint4 (&o)[8]) {
#pragma unroll
      for (int c = 0; c < 8; ++c) o[c] = *row_chunk(tile, r, c);
    };
    // dq = dy * z for tile i (z lane p = time 128 i + 127 - p); dy from stage ds.
    auto dq_tile = [&](int g, int i, int b, int ds, uint32_t dcount) -> bool {
      const int r = kTM - 1 - row_lane;
      const long long off = row_off(b, static_cast<long long>(i) * kTM + r, g);
      if (!tc::warp_wait(&bars[kBarDYFull + ds], (dcount / kNDY) & 1, abort)) return false;
      uint4 dr[8];
      smem_row(dy_st + ds * kTileBytes, r, dr);
      mbar_arrive(&bars[kBarDYEmpty + ds]);
      if (!tc::warp_wait(&bars[kBarZFull], zc & 1, abort)) return false;
      tc_fence_after_sync();
      uint32_t a0[32], a1[32];
      tmem_ld_32x32b_x32(tl + kColZ, a0);
      tmem_ld_32x32b_x32(tl + kColZ + 32, a1);
      tmem_wait_ld();
      reg_fence(a0);
      reg_fence(a1);
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarZEmpty]);
      ++zc;
      if (off >= 0) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.dq + off);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float d[8], o[8];
          unpack_bf16x8(dr[c], d);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = 8 * c + e;
            o[e] = d[e] * __uint_as_float(ch < 32 ? a0[ch] : a1[ch - 32]);
          }
          __stcs(dst + c, pack_bf16x8(o));
        }
      }
      return true;
    };
    bool ok = true;
    while (ok && it.next(t)) {
      if (t.kind == kNextHalo) {
        ++dc;
        continue;
      }
      if (t.kind == kMain) {
        // dk = dx * v and dv = dx * k (dx lane p = time 128 i + p)
        const int ks = kc % kNKV, ds = dc % kNDY;
        const uint32_t kcount = kc, dcount = dc;
        ++kc;
        ++dc;
        const long long off = row_off(t.b, static_cast<long long>(t.i) * kTM + row_lane, t.g);
        if (!tc::warp_wait(&bars[kBarKVFull + ks], (kcount / kNKV) & 1, abort)) break;
        uint4 kr[8], vr[8];
        uint8_t *ktile = kv_st + ks * 2 * kTileBytes;
        smem_row(ktile, row_lane, kr);
        smem_row(ktile + kTileBytes, row_lane, vr);
        mbar_arrive(&bars[kBarKVEmpty + ks]);
        if (!tc::warp_wait(&bars[kBarDXFull], dxc & 1, abort)) break;
        tc_fence_after_sync();
        uint32_t a0[32], a1[32];
        tmem_ld_32x32b_x32(tl + kColDX, a0);
        tmem_ld_32x32b_x32(tl + kColDX + 32, a1);
        tmem_wait_ld();
        reg_fence(a0);
        reg_fence(a1);
        tc_fence_before_sync();
        mbar_arrive(&bars[kBarDXEmpty]);
        ++dxc;
        if (off >= 0) {
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
        // dq of tile i + 1 (its z was issued with this tile)
        if (t.i < t.hi && !dq_tile(t.g, t.i + 1, t.b, prev_ds, prev_dc)) break;
        prev_ds = ds;
        prev_dc = dcount;
        continue;
      }
      // tail: dq of tile lo, then the dh sums of the segment
      if (t.lo > 0) ++kc;
      if (!dq_tile(t.g, t.lo, t.b, prev_ds, prev_dc)) break;
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
