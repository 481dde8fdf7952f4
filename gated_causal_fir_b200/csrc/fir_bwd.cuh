// fir_bwd.cuh -- CUDA-core kernels of the backward pass of the gated grouped causal FIR.
//
// For y = q * z, z = h_g conv x, x = k * v and an upstream gradient dy (page "04.
// Hardware-aware convolution kernels", Sec. 7 two-pass backward):
//   dq = dy * z              -- the forward kernels with dy in the place of q
//   dz = q * dy,  dx[t] = sum_j h[j] dz[t + j]   (transposed Toeplitz: anti-causal)
//   dk = dx * v,  dv = dx * k      -- cc::fir_tiled_kernel<T, true> (one pass, both outputs), or
//                                     fir_bwd_window_kernel below for short filters
//   dh[g][j] = sum_{b, t, c in g} dz[b,t,c] x[b,t-j,c]
//                            -- two passes as on the page: fir_bwd_dh_partial_kernel (or, for
//                               short filters, fir_bwd_window_kernel) writes partials, coalesced
//                               along j; fir_bwd_dh_reduce_kernel sums them in a fixed order.
// All arithmetic is fp32 with products formed before rounding (exact for bf16 inputs).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fir_cuda_core.cuh"

namespace hyena {
namespace bwd {

using cc::from_f32;
using cc::to_f32;

constexpr int kDhRows = 64;     // time rows of one partial
constexpr int kDhTaps = 128;    // taps per pass over the staged window (= threads per block)

// Channels per partial: the largest of 64, 32, ..., 1 that divides d_g (a piece never straddles
// two groups).
__host__ __device__ inline int dh_piece(int d_g) {
  int cp = 64;
  while (d_g % cp) cp >>= 1;
  return cp;
}

// Pass 1.  Block (chunk, piece, b): rows [64 chunk, 64 chunk + 64) of sequence b, channels
// [piece * cp, piece * cp + cp).  For each tap j of a 128-tap block it forms
//   sum_{t in rows, c in piece} dz[t, c] * x[t - j, c]
// from shared memory (the dz rows and the x window of the tap block, rows padded by one float)
// and writes partial[((b * nchunk + chunk) * npieces + piece) * l_h + j].  Thread (cg, tg) =
// (tid % 8, tid / 8) takes the 8 taps 8 tg .. 8 tg + 7 over the channels cg, cg + 8, ...: per 8
// rows of one channel it reads 8 dz values and 15 window values for 64 FMAs; the 8 channel
// groups' sums then meet in shared memory in a fixed order.
constexpr int kDhGroups = 8;                                  // channel groups per block
constexpr int kDhRedFloats = kDhGroups * kDhTaps;             // the reduction buffer

template <typename T>
__global__ void __launch_bounds__(kDhTaps)
    fir_bwd_dh_partial_kernel(const T *__restrict__ q, const T *__restrict__ k,
                              const T *__restrict__ v, const T *__restrict__ dy,
                              float *__restrict__ partial, long long L, long long D, int l_h,
                              int cp, int nchunk, int npieces, int B,
                              const unsigned *__restrict__ run_if, unsigned run_token) {
  if (run_if) {  // as fir_tiled_kernel's run_if
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (*run_if != run_token) return;
  }
  extern __shared__ float sm[];
  // one (chunk, piece, sequence) block after another, grid-stride
  const long long nblk = static_cast<long long>(nchunk) * npieces * B;
  for (long long blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
  const int chunk = static_cast<int>(blk % nchunk);
  const int piece = static_cast<int>((blk / nchunk) % npieces);
  const int b = static_cast<int>(blk / (static_cast<long long>(nchunk) * npieces));
  __syncthreads();  // the previous block's rows and sums have been read
  const long long t0 = static_cast<long long>(chunk) * kDhRows;
  const long long c0 = static_cast<long long>(piece) * cp;
  const long long base = static_cast<long long>(b) * L * D;
  const int ld = cp + 1;
  const int cg = threadIdx.x % kDhGroups, tg = threadIdx.x / kDhGroups;
  float *red = sm;                              // [kDhGroups][kDhTaps]
  float *dzs = sm + kDhRedFloats;               // [kDhRows][ld]
  float *xs = dzs + kDhRows * ld;               // [kDhRows + kDhTaps - 1][ld]
  for (int e = threadIdx.x; e < kDhRows * cp; e += blockDim.x) {
    const int r = e / cp, c = e % cp;
    const long long t = t0 + r;
    float val = 0.f;
    if (t < L) {
      const long long a = base + t * D + c0 + c;
      val = to_f32(q[a]) * to_f32(dy[a]);
    }
    dzs[r * ld + c] = val;
  }
  float *out = partial + ((static_cast<long long>(b) * nchunk + chunk) * npieces + piece) * l_h;
  for (int j0 = 0; j0 < l_h; j0 += kDhTaps) {
    // x rows t0 - j0 - (kDhTaps - 1) .. t0 + kDhRows - 1 - j0; window row w holds
    // x[t0 - j0 - (kDhTaps - 1) + w].
    const long long xbase = t0 - j0 - (kDhTaps - 1);
    __syncthreads();  // the previous tap block's window and reduction have been read
    for (int e = threadIdx.x; e < (kDhRows + kDhTaps - 1) * cp; e += blockDim.x) {
      const int w = e / cp, c = e % cp;
      const long long t = xbase + w;
      float val = 0.f;
      if (t >= 0 && t < L) {
        const long long a = base + t * D + c0 + c;
        val = to_f32(k[a]) * to_f32(v[a]);
      }
      xs[w * ld + c] = val;
    }
    __syncthreads();
    // dz row r pairs with window row r + (kDhTaps - 1) - jj for tap j0 + jj; for rows
    // r0 + i and taps 8 tg + t that is row w0 + (i - t + 7), w0 = r0 + kDhTaps - 8 - 8 tg
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    for (int c = cg; c < cp; c += kDhGroups) {
      for (int r0 = 0; r0 < kDhRows; r0 += 8) {
        const int w0 = r0 + kDhTaps - 8 - 8 * tg;
        float dz[8], xw[15];
#pragma unroll
        for (int i = 0; i < 8; ++i) dz[i] = dzs[(r0 + i) * ld + c];
#pragma unroll
        for (int u = 0; u < 15; ++u) xw[u] = xs[(w0 + u) * ld + c];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int t = 0; t < 8; ++t) acc[t] = fmaf(dz[i], xw[i - t + 7], acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) red[cg * kDhTaps + tg * 8 + t] = acc[t];
    __syncthreads();
    const int j = j0 + threadIdx.x;
    if (j < l_h) {
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < kDhGroups; ++g) s += red[g * kDhTaps + threadIdx.x];
      out[j] = s;
    }
  }
  }
}

// Short filters (l_h <= 16): dk, dv and the dh partials in one pass over q, k, v, dy, the
// backward counterpart of cc::fir_window_kernel.  A thread owns VN channels (16 bytes, all in one
// group) over a run of rows [t0, t1) and walks it in DECREASING time with a register window of
// dz = q dy over rows t .. t + l_h - 1 (the l_h - 1 rows after the run are its halo, zero past
// L):
//   dx[t] = sum_j h[j] dz[t + j]       (the transposed Toeplitz product, taps in order j = 0 ..)
//   dk[t] = dx[t] v[t],  dv[t] = dx[t] k[t]
//   dh[j] += sum_{c in thread} dz[t + j, c] x[t, c],  x = k v
// so every (t, j) pair of the filter gradient is met once, at the run that owns row t.  The
// thread's l_h partial sums go to partial[gid][j] (gid = (b n_tb + tb) cv + channel vector):
// the layout fir_bwd_dh_reduce_kernel reads with one piece per channel vector.
#ifndef HYENA_BWD_WINDOW_BLOCK
#define HYENA_BWD_WINDOW_BLOCK 128
#endif
constexpr int kBwdWindowBlock = HYENA_BWD_WINDOW_BLOCK;

template <typename T, int LH>
__global__ void __launch_bounds__(kBwdWindowBlock)
    fir_bwd_window_kernel(const T *__restrict__ q, const T *__restrict__ k,
                          const T *__restrict__ v, const float *__restrict__ h,
                          const T *__restrict__ dy, T *__restrict__ dk, T *__restrict__ dv,
                          float *__restrict__ partial, const cc::WindowParams p) {
  cc::pdl_enter();  // launched with programmatic stream serialisation
  using V = cc::Vec<T>;
  constexpr int VN = V::N;
  constexpr int U = LH <= 8 ? 4 : 2;  // rows of loads issued before their arithmetic
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= p.B * p.n_tb * p.cv) return;
  const long long cvi = gid % p.cv;
  const long long rest = gid / p.cv;
  const long long tb = rest % p.n_tb;
  const long long b = rest / p.n_tb;
  const long long c0 = cvi * VN;
  const long long g = c0 / p.d_g;

  float hr[LH];
#pragma unroll
  for (int j = 0; j < LH; ++j) hr[j] = __ldg(h + g * LH + j);
  float zw[LH][VN];  // zw[j] = dz at time t + j
  float dh[LH];
#pragma unroll
  for (int j = 0; j < LH; ++j) {
    dh[j] = 0.f;
#pragma unroll
    for (int e = 0; e < VN; ++e) zw[j][e] = 0.f;
  }
  const long long t0 = tb * p.rows;
  const long long t1 = min(t0 + p.rows, p.L);
  const long long seq = b * p.L * p.D + c0;

  // Halo: rows t1 + l_h - 2 down to t1 (zero from L on), so that the window is complete at the
  // first row of the run.
#pragma unroll
  for (int s = LH - 2; s >= 0; --s) {
#pragma unroll
    for (int j = LH - 1; j >= 1; --j)
#pragma unroll
      for (int e = 0; e < VN; ++e) zw[j][e] = zw[j - 1][e];
    const long long t = t1 + s;
    if (t < p.L) {
      float qq[VN], gg[VN];
      V::unpack(V::load(q + seq + t * p.D), qq);
      V::unpack(V::load(dy + seq + t * p.D), gg);
#pragma unroll
      for (int e = 0; e < VN; ++e) zw[0][e] = qq[e] * gg[e];
    } else {
#pragma unroll
      for (int e = 0; e < VN; ++e) zw[0][e] = 0.f;
    }
  }

  for (long long t = t1 - 1; t >= t0; t -= U) {
    uint4 qr[U], gr[U], kr[U], vr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (t - u >= t0) {
        const long long off = seq + (t - u) * p.D;
        qr[u] = V::load(q + off);
        gr[u] = V::load(dy + off);
        kr[u] = V::load(k + off);
        vr[u] = V::load(v + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (t - u >= t0) {
#pragma unroll
        for (int j = LH - 1; j >= 1; --j)
#pragma unroll
          for (int e = 0; e < VN; ++e) zw[j][e] = zw[j - 1][e];
        float qq[VN], gg[VN], kk[VN], vv[VN], ok[VN], ov[VN];
        V::unpack(qr[u], qq);
        V::unpack(gr[u], gg);
        V::unpack(kr[u], kk);
        V::unpack(vr[u], vv);
#pragma unroll
        for (int e = 0; e < VN; ++e) zw[0][e] = qq[e] * gg[e];
#pragma unroll
        for (int e = 0; e < VN; ++e) {
          float dx = 0.f;
#pragma unroll
          for (int j = 0; j < LH; ++j) dx = fmaf(hr[j], zw[j][e], dx);
          ok[e] = dx * vv[e];
          ov[e] = dx * kk[e];
          const float x = kk[e] * vv[e];
#pragma unroll
          for (int j = 0; j < LH; ++j) dh[j] = fmaf(zw[j][e], x, dh[j]);
        }
        const long long off = seq + (t - u) * p.D;
        V::store(dk + off, ok);
        V::store(dv + off, ov);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < LH; ++j) partial[gid * LH + j] = dh[j];
}

// Pass 2.  dh[g][j] = sum over b, chunk and the group's pieces of the partials.  One warp per
// output: lane i adds the terms i, i + 32, ... (term = (b, chunk, piece), piece fastest) in
// that order, then the 32 lane sums meet in a fixed butterfly (IEEE addition is commutative, so
// every lane ends with the same bits): deterministic, and the G l_h outputs spread over
// G l_h warps instead of as many threads.
constexpr int kReduceBlock = 256;
__global__ void __launch_bounds__(kReduceBlock)
    fir_bwd_dh_reduce_kernel(const float *__restrict__ partial, float *__restrict__ dh, int B,
                             int nchunk, int npieces, int pieces_per_group, int G, int l_h,
                             const unsigned *__restrict__ run_if, unsigned run_token) {
  if (run_if) {  // as fir_tiled_kernel's run_if
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (*run_if != run_token) return;
  }
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (kReduceBlock / 32);
  const long long n = static_cast<long long>(G) * l_h;
  const int terms = B * nchunk * pieces_per_group;  // < 2^31 (checked by the host)
  for (long long w = static_cast<long long>(blockIdx.x) * (kReduceBlock / 32) + threadIdx.x / 32;
       w < n; w += warps) {
    const int g = static_cast<int>(w / l_h), j = static_cast<int>(w % l_h);
    const float *pg = partial + static_cast<long long>(g) * pieces_per_group * l_h + j;
    float s = 0.f;
    for (int i = lane; i < terms; i += 32) {
      const int pc = i % pieces_per_group, bc = i / pieces_per_group;  // bc = b nchunk + chunk
      s += pg[(static_cast<long long>(bc) * npieces + pc) * l_h];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) dh[w] = s;
  }
}

}  // namespace bwd
}  // namespace hyena
