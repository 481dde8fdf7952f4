// fir_fftblk.cuh -- single-pass block FFT forward of the gated grouped causal convolution for
// long filters (the Hyena-LI class of the StripedHyena 2 overview, Sec. 3 operator table: long
// filters evaluated by FFT convolution), with no workspace.
//
// Overlap-save: the sequence is cut into time blocks of M = N - l_h + 1 outputs.  Block tb
// reads the N rows t = t0 - (l_h - 1) + r, r < N, t0 = tb M (rows before 0 are zero or come
// from the history tensors, rows past L are zero), and the length-N cyclic convolution of those
// rows with the zero-padded filter equals the causal sum (page "04. Hardware-aware convolution
// kernels", Sec. 1) at every r >= l_h - 1, i.e. at t0 .. t0 + M - 1: those are the rows kept.
//
// One CTA holds the N rows of P channel pairs in shared memory, each pair as one complex
// signal x_c + i x_{c+1} (both real, one filter: the inverse transform of H X is y_c + i y_{c+1}
// exactly).  The transform runs in place: a decimation-in-frequency FFT (a radix 2..16 stage,
// then radix-16 stages; each stage a DFT over R points in registers, times W_{RS}^{j k}) leaves
// the spectrum in digit-reversed order; it is multiplied there by the filter spectrum, which
// the same stages produced in the same order, and the mirror-image decimation-in-time stages
// bring the product back to natural order.  So no reordering pass is needed, and the middle
// stage (span 1) runs forward DFT, product and inverse DFT on the same registers.  1/N is
// folded into the filter spectrum.
//
// Each CTA (one per SM, persistent) walks a contiguous range of items (sequence b, channel
// block, time block), ordered so that consecutive items share the channel block and hence the
// group: the filter spectrum is transformed again only when the group changes.  Loads are
// software-pipelined through shared memory with cp.async: the next item's k and v rows are
// copied while the current item is transformed, and the current item's q rows while its
// forward transform runs.  The first stage reads k and v from there and forms x = k v on the
// way in; the last inverse stage multiplies by q and writes y to global memory directly.
// Q sibling CTAs (consecutive block indices) walk the same range in step, on Q consecutive
// channel blocks: together they read whole 64-byte pieces of each row at the same time, where
// one CTA alone would use 4P bytes (bf16) of every 64 that DRAM delivers.  Shared-memory rows
// of 16 complex values are padded to 18, so that every stage's 64-bit accesses and the middle
// stage's 128-bit row accesses are free of bank conflicts.  All arithmetic is fp32; q, k, v, y
// are bf16 or fp32.  The kernel launches with programmatic stream serialisation.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fir_fft.cuh"

namespace hyena {
namespace fftblk {

using fft::cconj;
using fft::cmul;
using fft::dft_reg;
using fft::ilog2;

constexpr int kRow = 18;  // complex slots per 16-point row of shared memory (2 of padding)

__host__ __device__ constexpr int sig_slots(int n) { return n / 16 * kRow; }
__device__ __forceinline__ int slot(int e) { return (e >> 4) * kRow + (e & 15); }

// Stages of a length-2^LGN transform: a first stage of radix R0 = 2^LG0 (span N / R0), then
// NS16 radix-16 stages of spans N / (R0 16^i); the last of them (span 1) is the middle stage.
template <int LGN>
struct Plan {
  static constexpr int N = 1 << LGN;
  static constexpr int LG0 = LGN % 4 == 0 ? 4 : LGN % 4;
  static constexpr int R0 = 1 << LG0;
  static constexpr int NS16 = (LGN - LG0) / 4;
  static_assert(NS16 >= 1, "at least one radix-16 stage");
};

// Shared memory of one CTA: P signals, the filter spectrum, the quarter twiddle table, the
// staged k and v rows of one item (row-major, RB bytes per row), and its q rows (kStageQ).
template <typename T, int LGN, int P, bool kStageQ>
struct Smem {
  static constexpr int N = 1 << LGN;
  static constexpr int kSig = sig_slots(N);
  static constexpr int RB = 2 * P * static_cast<int>(sizeof(T));
  static constexpr int kOffH = P * kSig * 8;
  static constexpr int kOffTw = kOffH + kSig * 8;
  static constexpr int kOffKV = kOffTw + N / 4 * 8;
  static constexpr int kOffQ = kOffKV + 2 * N * RB;
  static constexpr int kBytes = kOffQ + (kStageQ ? N * RB : 0);
};

struct BlkParams {
  const void *q, *k, *v, *kh, *vh;  // kh, vh: [B, Lh, D] rows before row 0 (Lh = 0: zeros)
  const float *h;
  void *y;
  long long L, D, Lh;
  long long items;  // B * (CB / Q) * nTB: the items of one CTA of each sibling group
  int CB;           // channel blocks per row (D / 2P)
  int Q;            // sibling CTAs: consecutive blocks that take consecutive channel blocks
  int nTB;          // time blocks per sequence (ceil(L / M))
  int M;            // outputs per block (N - l_h + 1)
  int d_g, l_h;
};

// W_N^e, 0 <= e < N, from the table tw[r] = W_N^r, r < N / 4: W_N^e = W_N^r (-i)^(e / (N/4)).
template <int LGN>
__device__ __forceinline__ float2 w_n(const float2 *tw, int e) {
  float2 w = tw[e & ((1 << (LGN - 2)) - 1)];
  const int quad = (e >> (LGN - 2)) & 3;
  if (quad & 2) w = make_float2(-w.x, -w.y);
  if (quad & 1) w = make_float2(w.y, -w.x);
  return w;
}

__host__ __device__ constexpr int high_bit(int k) {
  return k >= 8 ? 8 : (k >= 4 ? 4 : (k >= 2 ? 2 : 1));
}

// The twiddle powers W_{RS}^{j k} (or their conjugates), k = 1 .. R-1, of one task: by squaring
// and products (at most five rounded products deep; R <= 16).
template <int R, bool kConj>
__device__ __forceinline__ void twiddle_powers(float2 (&pw)[R], float2 w) {
  if (kConj) w = cconj(w);
  pw[0] = make_float2(1.f, 0.f);
  if constexpr (R > 1) pw[1] = w;
#pragma unroll
  for (int k = 2; k < R; ++k) {
    const int hi = high_bit(k);  // compile-time after unrolling
    pw[k] = hi == k ? cmul(pw[k / 2], pw[k / 2]) : cmul(pw[hi], pw[k - hi]);
  }
}

// One stage of radix R and span S = 2^LGS over `nsig` signals (signal stride kSig): for every
// block and j < S, the R points j + S m, a DFT over m, and (forward) times W_{RS}^{j k}
// afterwards or (inverse) times W_{RS}^{-j k} before.  A thread takes one (block, j) task at a
// time and runs it on every signal it owns, so the twiddles are formed once per task.  For
// S >= 16 the R points lie (S / 16) padded rows apart: a constant stride in shared memory.
template <int LGN, int R, int LGS, bool kInv>
__device__ __forceinline__ void stage(float2 *buf, int nsig, const float2 *tw, int tid, int nt) {
  constexpr int LGR = ilog2(R), S = 1 << LGS, kSig = sig_slots(1 << LGN);
  constexpr int TPS = (1 << LGN) / R;       // tasks per signal
  constexpr int TWS = LGN - LGR - LGS;      // W_{RS} = W_N^(2^TWS)
  static_assert(S >= 16, "the span-1 stage is the middle stage");
  constexpr int kStride = S / 16 * kRow;    // slots between the task's points
  // nt and TPS are powers of two: either every thread owns one task and a share of the
  // signals, or every thread owns several tasks and all signals
  const int sig0 = nt >= TPS ? tid / TPS : 0, sig_step = nt >= TPS ? nt / TPS : 1;
  const int task_step = nt >= TPS ? TPS : nt;
  for (int task = nt >= TPS ? tid % TPS : tid; task < TPS; task += task_step) {
    const int j = task & (S - 1), blk = task >> LGS;
    const int sb = slot((blk << (LGR + LGS)) + j);
    float2 pw[R];
    twiddle_powers<R, kInv>(pw, w_n<LGN>(tw, j << TWS));
    for (int sig = sig0; sig < nsig; sig += sig_step) {
      float2 *b = buf + sig * kSig + sb;
      float2 v[R];
#pragma unroll
      for (int m = 0; m < R; ++m) v[m] = b[m * kStride];
      if constexpr (kInv) {
#pragma unroll
        for (int m = 1; m < R; ++m) v[m] = cmul(v[m], pw[m]);
      }
      dft_reg<R, kInv>(v);
      if constexpr (!kInv) {
#pragma unroll
        for (int m = 1; m < R; ++m) v[m] = cmul(v[m], pw[m]);
      }
#pragma unroll
      for (int m = 0; m < R; ++m) b[m * kStride] = v[m];
    }
  }
}

// The forward stages before the middle one, each followed by a CTA barrier.
template <int LGN>
__device__ __forceinline__ void forward_outer(float2 *buf, int nsig, const float2 *tw, int tid,
                                              int nt) {
  using PL = Plan<LGN>;
  stage<LGN, PL::R0, LGN - PL::LG0, false>(buf, nsig, tw, tid, nt);
  __syncthreads();
  if constexpr (PL::NS16 >= 2) {
    stage<LGN, 16, LGN - PL::LG0 - 4, false>(buf, nsig, tw, tid, nt);
    __syncthreads();
  }
  if constexpr (PL::NS16 >= 3) {
    stage<LGN, 16, LGN - PL::LG0 - 8, false>(buf, nsig, tw, tid, nt);
    __syncthreads();
  }
  static_assert(PL::NS16 <= 3, "transform length");
}

__device__ __forceinline__ void load_row16(const float2 *row, float2 (&v)[16]) {
  const float4 *r4 = reinterpret_cast<const float4 *>(row);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = r4[i];
    v[2 * i] = make_float2(f.x, f.y);
    v[2 * i + 1] = make_float2(f.z, f.w);
  }
}
__device__ __forceinline__ void store_row16(float2 *row, const float2 (&v)[16]) {
  float4 *r4 = reinterpret_cast<float4 *>(row);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    r4[i] = make_float4(v[2 * i].x, v[2 * i].y, v[2 * i + 1].x, v[2 * i + 1].y);
}

// The middle stage (radix 16, span 1) on the data: forward DFT, times the filter spectrum,
// inverse DFT, on the same registers.  Without kData (the filter itself) only the forward DFT.
template <int LGN, bool kData>
__device__ __forceinline__ void middle(float2 *buf, int nsig, const float2 *Hs, int tid, int nt) {
  constexpr int LGT = LGN - 4, kSig = sig_slots(1 << LGN);
  const int total = nsig << LGT;
  for (int tk = tid; tk < total; tk += nt) {
    const int sig = tk >> LGT, blk = tk & ((1 << LGT) - 1);
    float2 *row = buf + sig * kSig + blk * kRow;
    float2 v[16];
    load_row16(row, v);
    dft_reg<16, false>(v);
    if constexpr (kData) {
      float2 hv[16];
      load_row16(Hs + blk * kRow, hv);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = cmul(v[i], hv[i]);
      dft_reg<16, true>(v);
    }
    store_row16(row, v);
  }
}

// cp.async of `bytes` (4, 8 or 16) from global to shared memory; src_bytes = 0 fills zeros.
template <int kBytes>
__device__ __forceinline__ void cp_async(void *dst, const void *src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const int n = valid ? kBytes : 0;
  if constexpr (kBytes == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(d), "l"(src), "n"(kBytes), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copies one row of RB bytes (a channel block of one tensor) in pieces of at most 16 bytes.
template <int RB>
__device__ __forceinline__ void copy_row(uint8_t *dst, const uint8_t *src, bool valid) {
  if constexpr (RB >= 16) {
#pragma unroll
    for (int i = 0; i < RB / 16; ++i) cp_async<16>(dst + 16 * i, src + 16 * i, valid);
  } else {
    cp_async<RB>(dst, src, valid);
  }
}

// Loads `kB` bytes (4, 8 or 16) of shared memory as 32-bit words.
template <int kB>
__device__ __forceinline__ void lds_words(const uint8_t *p, uint32_t (&w)[kB / 4]) {
  if constexpr (kB == 16) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
  } else if constexpr (kB == 8) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    w[0] = u.x, w[1] = u.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t *>(p);
  }
}
template <int kB>
__device__ __forceinline__ void ldg_words(const uint8_t *p, uint32_t (&w)[kB / 4]) {
  if constexpr (kB == 16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
  } else if constexpr (kB == 8) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    w[0] = u.x, w[1] = u.y;
  } else {
    w[0] = __ldg(reinterpret_cast<const unsigned int *>(p));
  }
}
template <int kB>
__device__ __forceinline__ void stg_words(uint8_t *p, const uint32_t (&w)[kB / 4]) {
  if constexpr (kB == 16)
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  else if constexpr (kB == 8)
    *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
  else
    *reinterpret_cast<uint32_t *>(p) = w[0];
}

// n values of T packed in 32-bit words, widened to fp32, and back (RNE for bf16).
template <typename T, int n>
__device__ __forceinline__ void unpack(const uint32_t *w, float (&o)[n]) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < n; ++i) o[i] = __uint_as_float(w[i]);
  }
}
template <typename T, int n>
__device__ __forceinline__ void pack(const float (&o)[n], uint32_t *w) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
  } else {
#pragma unroll
    for (int i = 0; i < n; ++i) w[i] = __float_as_uint(o[i]);
  }
}

// The split of the first and last stages: N / R0 tasks, each over the P signals of the CTA;
// where there are more threads than tasks, SPLIT threads share a task, PS signals each.
template <int LGN, int P, int NT>
struct Outer {
  static constexpr int R0 = Plan<LGN>::R0, LGS0 = LGN - Plan<LGN>::LG0;
  static constexpr int TPS = (1 << LGN) / R0;
  static constexpr int SPLIT = NT >= TPS ? (NT / TPS < P ? NT / TPS : P) : 1;
  static constexpr int PS = P / SPLIT;
  static constexpr int kStride = (1 << LGS0) / 16 * kRow;
};

// Item coordinates: sequence, first channel of the block, time of row 0 of the block.
struct Item {
  long long b, ch0, t0;
  int g, tb;
};

template <typename T, int LGN, int P, int NT, bool kStageQ>
__global__ void __launch_bounds__(NT, 1) fir_fftblk_kernel(const BlkParams p) {
  constexpr int N = 1 << LGN, kSig = sig_slots(N);
  using SM = Smem<T, LGN, P, kStageQ>;
  using OU = Outer<LGN, P, NT>;
  constexpr int RB = SM::RB;                                  // bytes of a row piece
  constexpr int CH = OU::PS * 2 * static_cast<int>(sizeof(T));  // bytes a thread takes of it
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float2 *data = reinterpret_cast<float2 *>(smem_raw);        // [P][kSig]
  float2 *Hs = reinterpret_cast<float2 *>(smem_raw + SM::kOffH);
  float2 *tw = reinterpret_cast<float2 *>(smem_raw + SM::kOffTw);
  uint8_t *kst = smem_raw + SM::kOffKV, *vst = kst + N * RB;  // staged k, v rows
  uint8_t *qst = smem_raw + SM::kOffQ;                        // staged q rows
  const int tid = threadIdx.x;
  for (int r = tid; r < N / 4; r += NT) tw[r] = fft::twiddle(r, N);
  // Launched with programmatic stream serialisation: the next kernel of the stream may be
  // scheduled at once, and this one reads no global memory before the previous kernel has
  // completed (the twiddle table above overlaps its tail).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const uint8_t *q = static_cast<const uint8_t *>(p.q), *k = static_cast<const uint8_t *>(p.k),
                *v = static_cast<const uint8_t *>(p.v), *kh = static_cast<const uint8_t *>(p.kh),
                *vh = static_cast<const uint8_t *>(p.vh);
  uint8_t *y = static_cast<uint8_t *>(p.y);
  constexpr long long ES = sizeof(T);
  const long long SG = gridDim.x / p.Q, c = blockIdx.x / p.Q;
  const int sib = static_cast<int>(blockIdx.x % p.Q);
  const long long i0 = c * p.items / SG, i1 = (c + 1) * p.items / SG;
  const long long per_b = static_cast<long long>(p.CB / p.Q) * p.nTB;
  const float inv_n = 1.0f / static_cast<float>(N);
  auto item = [&](long long it) {
    Item o;
    o.b = it / per_b;
    const int rem = static_cast<int>(it - o.b * per_b);
    const int cq = rem / p.nTB;
    o.tb = rem - cq * p.nTB;
    o.ch0 = static_cast<long long>(cq * p.Q + sib) * 2 * P;
    o.g = static_cast<int>(o.ch0 / p.d_g);
    o.t0 = static_cast<long long>(o.tb) * p.M - (p.l_h - 1);
    return o;
  };
  // k and v rows of an item into the staging rows (zero outside the sequence and history)
  auto stage_kv = [&](const Item &o) {
    for (int r = tid; r < N; r += NT) {
      const long long t = o.t0 + r;
      const bool main = t >= 0 && t < p.L, hist = t < 0 && t >= -p.Lh;
      const long long off = main ? ((o.b * p.L + t) * p.D + o.ch0) * ES
                                 : (hist ? ((o.b * p.Lh + p.Lh + t) * p.D + o.ch0) * ES : 0);
      copy_row<RB>(kst + r * RB, (hist ? kh : k) + off, main || hist);
      copy_row<RB>(vst + r * RB, (hist ? vh : v) + off, main || hist);
    }
  };
  // q rows of an item that hold outputs (r >= l_h - 1, t < L)
  auto stage_q = [&](const Item &o) {
    if constexpr (kStageQ) {
      for (int r = p.l_h - 1 + tid; r < N; r += NT) {
        const long long t = o.t0 + r;
        if (t >= p.L) break;
        copy_row<RB>(qst + r * RB, q + ((o.b * p.L + t) * p.D + o.ch0) * ES, true);
      }
    }
  };

  if (i0 < i1) {
    const Item o = item(i0);
    stage_kv(o);
    cp_async_commit();
    stage_q(o);
    cp_async_commit();
  }
  int cur_g = -1;
  for (long long it = i0; it < i1; ++it) {
    const Item o = item(it);
    if (o.g != cur_g) {  // the group's filter spectrum (1/N folded in), digit-reversed order
      __syncthreads();   // the table is written; the previous spectrum is no longer read
      const float *hg = p.h + static_cast<long long>(o.g) * p.l_h;
      for (int r = tid; r < N; r += NT)
        Hs[slot(r)] = make_float2(r < p.l_h ? __ldg(hg + r) * inv_n : 0.f, 0.f);
      __syncthreads();
      forward_outer<LGN>(Hs, 1, tw, tid, NT);
      middle<LGN, false>(Hs, 1, nullptr, tid, NT);
      cur_g = o.g;
    }
    cp_async_wait<1>();  // this item's k, v (its q may still be in flight)
    __syncthreads();
    // first stage, radix R0 over span N / R0, from the staged rows: x = k v per channel pair
    for (int task = NT >= OU::TPS ? tid % OU::TPS : tid; task < OU::TPS;
         task += NT >= OU::TPS ? OU::TPS : NT) {
      const int part = NT >= OU::TPS ? tid / OU::TPS : 0;
      if (part >= OU::SPLIT) break;
      float x[OU::R0][2 * OU::PS];
#pragma unroll
      for (int m = 0; m < OU::R0; ++m) {
        const int r = task + (m << OU::LGS0);
        uint32_t kw[CH / 4], vw[CH / 4];
        lds_words<CH>(kst + r * RB + part * CH, kw);
        lds_words<CH>(vst + r * RB + part * CH, vw);
        float kf[2 * OU::PS], vf[2 * OU::PS];
        unpack<T, 2 * OU::PS>(kw, kf);
        unpack<T, 2 * OU::PS>(vw, vf);
#pragma unroll
        for (int i = 0; i < 2 * OU::PS; ++i) x[m][i] = kf[i] * vf[i];
      }
      float2 pw[OU::R0];
      twiddle_powers<OU::R0, false>(pw, w_n<LGN>(tw, task));
      const int sb = slot(task);
#pragma unroll
      for (int s = 0; s < OU::PS; ++s) {
        float2 z[OU::R0];
#pragma unroll
        for (int m = 0; m < OU::R0; ++m) z[m] = make_float2(x[m][2 * s], x[m][2 * s + 1]);
        dft_reg<OU::R0, false>(z);
        float2 *bsig = data + (part * OU::PS + s) * kSig + sb;
#pragma unroll
        for (int m = 0; m < OU::R0; ++m) bsig[m * OU::kStride] = m ? cmul(z[m], pw[m]) : z[m];
      }
    }
    __syncthreads();  // the staged k, v rows are consumed
    if (it + 1 < i1) stage_kv(item(it + 1));
    cp_async_commit();
    using PL = Plan<LGN>;
    if constexpr (PL::NS16 >= 2) {
      stage<LGN, 16, LGN - PL::LG0 - 4, false>(data, P, tw, tid, NT);
      __syncthreads();
    }
    if constexpr (PL::NS16 >= 3) {
      stage<LGN, 16, LGN - PL::LG0 - 8, false>(data, P, tw, tid, NT);
      __syncthreads();
    }
    middle<LGN, true>(data, P, Hs, tid, NT);
    __syncthreads();
    if constexpr (PL::NS16 >= 3) {
      stage<LGN, 16, LGN - PL::LG0 - 8, true>(data, P, tw, tid, NT);
      __syncthreads();
    }
    if constexpr (PL::NS16 >= 2) {
      stage<LGN, 16, LGN - PL::LG0 - 4, true>(data, P, tw, tid, NT);
      __syncthreads();
    }
    cp_async_wait<1>();  // this item's q (the next item's k, v may still be in flight)
    __syncthreads();
    // last stage, inverse radix R0: rows r >= l_h - 1 hold the causal sum at t = t0 + r,
    // y = q * conv for t < L, written straight to global memory
    for (int task = NT >= OU::TPS ? tid % OU::TPS : tid; task < OU::TPS;
         task += NT >= OU::TPS ? OU::TPS : NT) {
      const int part = NT >= OU::TPS ? tid / OU::TPS : 0;
      if (part >= OU::SPLIT) break;
      float2 pw[OU::R0];
      twiddle_powers<OU::R0, true>(pw, w_n<LGN>(tw, task));
      const int sb = slot(task);
      float out[OU::R0][2 * OU::PS];
#pragma unroll
      for (int s = 0; s < OU::PS; ++s) {
        const float2 *bsig = data + (part * OU::PS + s) * kSig + sb;
        float2 z[OU::R0];
#pragma unroll
        for (int m = 0; m < OU::R0; ++m) z[m] = m ? cmul(bsig[m * OU::kStride], pw[m]) : bsig[0];
        dft_reg<OU::R0, true>(z);
#pragma unroll
        for (int m = 0; m < OU::R0; ++m) out[m][2 * s] = z[m].x, out[m][2 * s + 1] = z[m].y;
      }
#pragma unroll
      for (int m = 0; m < OU::R0; ++m) {
        const int r = task + (m << OU::LGS0);
        const long long t = o.t0 + r;
        if (r < p.l_h - 1 || t >= p.L) continue;
        const long long goff = ((o.b * p.L + t) * p.D + o.ch0) * ES + part * CH;
        uint32_t qw[CH / 4];
        if constexpr (kStageQ)
          lds_words<CH>(qst + r * RB + part * CH, qw);
        else
          ldg_words<CH>(q + goff, qw);
        float qf[2 * OU::PS];
        unpack<T, 2 * OU::PS>(qw, qf);
#pragma unroll
        for (int i = 0; i < 2 * OU::PS; ++i) qf[i] *= out[m][i];
        uint32_t yw[CH / 4];
        pack<T, 2 * OU::PS>(qf, yw);
        stg_words<CH>(y + goff, yw);
      }
    }
    __syncthreads();  // the staged q rows and the signals are consumed
    if (it + 1 < i1) stage_q(item(it + 1));
    cp_async_commit();
  }
  cp_async_wait<0>();
}

}  // namespace fftblk
}  // namespace hyena
