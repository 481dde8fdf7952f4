// fir_cuda_core.cuh -- CUDA-core kernels of the gated grouped causal FIR.
//
//  * fir_window_kernel: register sliding window for short filters (l_h <= 16, the Hyena-SE
//    class of the StripedHyena 2 overview, Sec. 3 operator table).  Each thread owns 16 bytes of
//    channels (8 bf16 or 4 fp32, all in one group) over a run of consecutive time steps and
//    keeps the last l_h values of x = k*v in registers, so every input is loaded from global
//    memory once per run (plus an l_h - 1 row halo) and the output is written once.  This is the
//    direct causal sum of page "04. Hardware-aware convolution kernels", Sec. 1, evaluated
//    output by output; for l_h <= 16 it needs ~2 l_h flops per element, far below the HBM
//    roofline's compute ridge, so no GEMM is needed.
//  * fir_direct_kernel: one thread per output element, taps read through the cache; any
//    supported shape, any alignment.  The fallback for shapes the fast kernels do not cover.
//
// Both accumulate in fp32 in tap order j = 0 .. l_h-1; x = k*v is formed in fp32 (exact for
// bf16 inputs) and y = q * acc is rounded once to the output type.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace hyena {
namespace cc {

template <typename T>
struct Vec;  // 16-byte vector of T

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static uint4 load(const __nv_bfloat16 *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
  }
  __device__ static void unpack(const uint4 &u, float (&o)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static void store(__nv_bfloat16 *p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static uint4 load(const float *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
  }
  __device__ static void unpack(const uint4 &u, float (&o)[4]) {
    o[0] = __uint_as_float(u.x);
    o[1] = __uint_as_float(u.y);
    o[2] = __uint_as_float(u.z);
    o[3] = __uint_as_float(u.w);
  }
  __device__ static void store(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ void from_f32(float v, __nv_bfloat16 *p) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void from_f32(float v, float *p) { *p = v; }

struct WindowParams {
  long long B, L, D;
  int d_g;
  int rows;        // time steps per thread
  long long n_tb;  // time blocks per sequence = ceil(L / rows)
  long long cv;    // channel vectors per row = D / VEC
  const void *kh, *vh;  // [B, Lh, D]: the rows before row 0 of every sequence (Lh = 0: zeros)
  long long Lh;
};

// Unroll factor of the time loop: loads of U rows are issued before their arithmetic.
#ifndef HYENA_WINDOW_UNROLL
#define HYENA_WINDOW_UNROLL 4
#endif
constexpr int kWindowUnroll = HYENA_WINDOW_UNROLL;

#ifndef HYENA_WINDOW_BLOCK
#define HYENA_WINDOW_BLOCK 128
#endif
#ifndef HYENA_WINDOW_MIN_BLOCKS
#define HYENA_WINDOW_MIN_BLOCKS 1
#endif
constexpr int kWindowBlock = HYENA_WINDOW_BLOCK;

template <typename T, int LH>
__global__ void __launch_bounds__(kWindowBlock, HYENA_WINDOW_MIN_BLOCKS)
    fir_window_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const float *__restrict__ h, T *__restrict__ y, const WindowParams p) {
  constexpr int VN = Vec<T>::N;
  // Longer windows hold more registers: they unroll no further than 4 rows.
  constexpr int U = LH <= 8 ? kWindowUnroll : (kWindowUnroll < 4 ? kWindowUnroll : 4);
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

  float xw[LH][VN];  // xw[j] = x at time t - j
#pragma unroll
  for (int j = 0; j < LH; ++j)
#pragma unroll
    for (int e = 0; e < VN; ++e) xw[j][e] = 0.f;

  const long long t0 = tb * p.rows;
  const long long t_end = min(t0 + p.rows, p.L);
  const long long seq = b * p.L * p.D + c0;

  // Halo: the l_h - 1 rows before t0 (before row 0: the history rows, then zeros).
#pragma unroll
  for (int s = LH - 1; s >= 1; --s) {
#pragma unroll
    for (int j = LH - 1; j >= 1; --j)
#pragma unroll
      for (int e = 0; e < VN; ++e) xw[j][e] = xw[j - 1][e];
    const long long t = t0 - s;
    if (t >= -p.Lh) {
      const T *kp = t >= 0 ? k + seq + t * p.D
                           : static_cast<const T *>(p.kh) + (b * p.Lh + p.Lh + t) * p.D + c0;
      const T *vp = t >= 0 ? v + seq + t * p.D
                           : static_cast<const T *>(p.vh) + (b * p.Lh + p.Lh + t) * p.D + c0;
      float kk[VN], vv[VN];
      Vec<T>::unpack(Vec<T>::load(kp), kk);
      Vec<T>::unpack(Vec<T>::load(vp), vv);
#pragma unroll
      for (int e = 0; e < VN; ++e) xw[0][e] = kk[e] * vv[e];
    } else {
#pragma unroll
      for (int e = 0; e < VN; ++e) xw[0][e] = 0.f;
    }
  }

  for (long long t = t0; t < t_end; t += U) {
    uint4 kr[U], vr[U], qr[U];  // packed rows, unpacked at use
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (t + u < t_end) {
        const long long off = seq + (t + u) * p.D;
        kr[u] = Vec<T>::load(k + off);
        vr[u] = Vec<T>::load(v + off);
        qr[u] = Vec<T>::load(q + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (t + u < t_end) {
#pragma unroll
        for (int j = LH - 1; j >= 1; --j)
#pragma unroll
          for (int e = 0; e < VN; ++e) xw[j][e] = xw[j - 1][e];
        float kk[VN], vv[VN], qq[VN];
        Vec<T>::unpack(kr[u], kk);
        Vec<T>::unpack(vr[u], vv);
        Vec<T>::unpack(qr[u], qq);
#pragma unroll
        for (int e = 0; e < VN; ++e) xw[0][e] = kk[e] * vv[e];
        float out[VN];
#pragma unroll
        for (int e = 0; e < VN; ++e) {
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < LH; ++j) acc = fmaf(hr[j], xw[j][e], acc);
          out[e] = qq[e] * acc;
        }
        Vec<T>::store(y + seq + (t + u) * p.D, out);
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
    fir_direct_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const float *__restrict__ h, T *__restrict__ y, long long B, long long L,
                      long long D, int d_g, int l_h, const T *__restrict__ kh,
                      const T *__restrict__ vh, long long Lh) {
  const long long n = B * L * D;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e % D;
    const long long t = (e / D) % L;
    const float *hg = h + (c / d_g) * l_h;
    const long long jmax = min(static_cast<long long>(l_h - 1), t);
    float acc = 0.f;
    for (long long j = 0; j <= jmax; ++j) {
      const long long src = e - j * D;
      acc = fmaf(__ldg(hg + j), to_f32(k[src]) * to_f32(v[src]), acc);
    }
    // taps that reach before row 0: the history rows [B, Lh, D] (row Lh - 1 precedes row 0)
    const long long jh = min(static_cast<long long>(l_h - 1), t + Lh);
    if (jh > t) {
      const long long hrow = (e / (L * D)) * Lh + Lh + t;  // history row of tap j: hrow - j
      for (long long j = t + 1; j <= jh; ++j) {
        const long long src = (hrow - j) * D + c;
        acc = fmaf(__ldg(hg + j), to_f32(kh[src]) * to_f32(vh[src]), acc);
      }
    }
    from_f32(to_f32(q[e]) * acc, y + e);
  }
}

// Toeplitz sub-blocks H_m[g][i][j] = h[g][m*l_b + i - j] (zero outside [0, l_h)), m = 0, 1, 2.
__global__ void __launch_bounds__(256)
    toeplitz_blocks_kernel(const float *__restrict__ h, float *H0, float *H1, float *H2, int G,
                           int l_h, int l_b) {
  const long long n = static_cast<long long>(G) * l_b * l_b;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long g = e / (static_cast<long long>(l_b) * l_b);
    const int i = static_cast<int>((e / l_b) % l_b);
    const int j = static_cast<int>(e % l_b);
    float *outs[3] = {H0, H1, H2};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      if (outs[m] == nullptr) continue;
      const int idx = m * l_b + i - j;
      outs[m][e] = (idx >= 0 && idx < l_h) ? __ldg(h + g * l_h + idx) : 0.f;
    }
  }
}

// All S sub-block diagonals: Hm[m][g][i][j] = h[g][m l_b + i - j] inside [0, l_h), else 0, for
// m < S (the general block form of the same page, any filter length).
__global__ void __launch_bounds__(256)
    toeplitz_stack_kernel(const float *__restrict__ h, float *__restrict__ Hm, int S, int G,
                          int l_h, int l_b) {
  const long long blk = static_cast<long long>(l_b) * l_b;
  const long long n = static_cast<long long>(S) * G * blk;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long mg = e / blk;
    const int m = static_cast<int>(mg / G);
    const long long g = mg % G;
    const int i = static_cast<int>((e / l_b) % l_b);
    const int j = static_cast<int>(e % l_b);
    const long long idx = static_cast<long long>(m) * l_b + i - j;
    Hm[e] = (idx >= 0 && idx < l_h) ? __ldg(h + g * l_h + idx) : 0.f;
  }
}

}  // namespace cc
}  // namespace hyena
