// fir_bwd.cuh -- CUDA-core kernels of the backward pass of the gated grouped causal FIR.
//
// For y = q * z, z = h_g conv x, x = k * v and an upstream gradient dy (page "04.
// Hardware-aware convolution kernels", Sec. 7 two-pass backward):
//   dq = dy * z              -- the forward kernels with dy in the place of q
//   dz = q * dy,  dx[t] = sum_j h[j] dz[t + j]   (transposed Toeplitz: anti-causal)
//   dk = dx * v,  dv = dx * k                      -- fir_bwd_dx_kernel (one pass, both outputs)
//   dh[g][j] = sum_{b, t, c in g} dz[b,t,c] x[b,t-j,c]
//                            -- two passes as on the page: fir_bwd_dh_partial_kernel writes one
//                               partial per (sequence, 64-row chunk, channel piece), coalesced
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

// dk, dv for every element: dx = sum_{j < l_h, t + j < L} h[g][j] * q[t+j] * dy[t+j].
template <typename T>
__global__ void __launch_bounds__(256)
    fir_bwd_dx_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const float *__restrict__ h, const T *__restrict__ dy, T *__restrict__ dk,
                      T *__restrict__ dv, long long B, long long L, long long D, int d_g,
                      int l_h) {
  const long long n = B * L * D;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e % D;
    const long long t = (e / D) % L;
    const float *hg = h + (c / d_g) * l_h;
    const long long jmax = min(static_cast<long long>(l_h - 1), L - 1 - t);
    float dx = 0.f;
    for (long long j = 0; j <= jmax; ++j) {
      const long long src = e + j * D;
      dx = fmaf(__ldg(hg + j), to_f32(q[src]) * to_f32(dy[src]), dx);
    }
    from_f32(dx * to_f32(v[e]), dk + e);
    from_f32(dx * to_f32(k[e]), dv + e);
  }
}

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
// [piece * cp, piece * cp + cp).  Thread j of a tap block accumulates
//   sum_{t in rows, c in piece} dz[t, c] * x[t - j, c]
// from shared memory (dz rows and the x window the tap block needs, rows padded by one float so
// that the lanes' different rows fall in different banks), and writes
// partial[((b * nchunk + chunk) * npieces + piece) * l_h + j].
template <typename T>
__global__ void __launch_bounds__(kDhTaps)
    fir_bwd_dh_partial_kernel(const T *__restrict__ q, const T *__restrict__ k,
                              const T *__restrict__ v, const T *__restrict__ dy,
                              float *__restrict__ partial, long long L, long long D, int l_h,
                              int cp) {
  extern __shared__ float sm[];
  const int chunk = blockIdx.x, piece = blockIdx.y, b = blockIdx.z;
  const int nchunk = gridDim.x, npieces = gridDim.y;
  const long long t0 = static_cast<long long>(chunk) * kDhRows;
  const long long c0 = static_cast<long long>(piece) * cp;
  const long long base = static_cast<long long>(b) * L * D;
  const int ld = cp + 1;
  float *dzs = sm;                       // [kDhRows][ld]
  float *xs = sm + kDhRows * ld;         // [kDhRows + kDhTaps - 1][ld]
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
    __syncthreads();
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
    const int j = j0 + threadIdx.x;
    float acc = 0.f;
    // row r of dz pairs with x row t0 + r - j = window row r + (kDhTaps - 1) - threadIdx.x
    const int woff = kDhTaps - 1 - static_cast<int>(threadIdx.x);
    for (int r = 0; r < kDhRows; ++r) {
      const float *dzr = dzs + r * ld;
      const float *xr = xs + (r + woff) * ld;
      for (int c = 0; c < cp; ++c) acc = fmaf(dzr[c], xr[c], acc);
    }
    if (j < l_h) out[j] = acc;
  }
}

// Pass 2.  dh[g][j] = sum over b, chunk and the group's pieces of the partials, in that order.
__global__ void __launch_bounds__(256)
    fir_bwd_dh_reduce_kernel(const float *__restrict__ partial, float *__restrict__ dh, int B,
                             int nchunk, int npieces, int pieces_per_group, int G, int l_h) {
  const long long n = static_cast<long long>(G) * l_h;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(e / l_h), j = static_cast<int>(e % l_h);
    float s = 0.f;
    for (int b = 0; b < B; ++b)
      for (int ch = 0; ch < nchunk; ++ch) {
        const float *row = partial + ((static_cast<long long>(b) * nchunk + ch) * npieces +
                                      static_cast<long long>(g) * pieces_per_group) * l_h + j;
        for (int pc = 0; pc < pieces_per_group; ++pc) s += row[static_cast<long long>(pc) * l_h];
      }
    dh[e] = s;
  }
}

}  // namespace bwd
}  // namespace hyena
