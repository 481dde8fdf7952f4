// fir_fft.cuh -- FFT kernels of the gated grouped causal convolution for long filters (the
// Hyena-LI class of the StripedHyena 2 overview, Sec. 3 operator table: long implicit filters,
// evaluated by FFT convolution, O(L log L) per channel instead of O(L l_h)).
//
// The convolution y = q * (h_g conv x), x = k * v, is evaluated as a cyclic convolution of
// length N = N1 N2 >= L + l_h - 1 (a power of two): zero padding makes the cyclic sum equal
// the causal one for every t < L.  The length-N DFT uses the four-step factorisation
//     X[k1 + N1 k2] = sum_{n2} W_N2^{n2 k2} W_N^{n2 k1} sum_{n1} x[N2 n1 + n2] W_N1^{n1 k1},
// W_M = exp(-2 pi i / M), and its inverse in the mirrored order.  Three kernels:
//   pass 1 (per n2): x = k v over the rows t = N2 n1 + n2, length-N1 FFT, times W_N^{n2 k1};
//   pass 2 (per k1): length-N2 FFT, times the filter spectrum H[k1 + N1 k2], inverse FFT;
//   pass 3 (per n2): times W_N^{-n2 k1}, inverse length-N1 FFT, / N, times q, store t < L.
// The filter spectrum comes from passes 1 and 2 run on h ("spectrum" mode).
//
// Two channels of one group travel as one complex signal x_c + i x_{c+1}: their filter (and
// so its spectrum) is the same and both signals are real, so the inverse transform of
// H (X_c + i X_{c+1}) is y_c + i y_{c+1} exactly -- no separation step.
//
// Every FFT runs in shared memory: P signals (channel pairs) side by side, radix-4 (and one
// radix-2) Stockham stages (self-sorting: natural order in, natural order out), twiddles from
// sincospif tabled once per CTA.  The
// intermediate spectra live in a caller-owned fp32 workspace laid out [b][k1][n2][pair], so
// every pass reads and writes P contiguous complex values (128 bytes) per index.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fir_cuda_core.cuh"

namespace hyena {
namespace fft {

constexpr int kP = 16;          // signals (channel pairs) per CTA
constexpr int kThreads = 256;
constexpr int kMaxLen = 256;    // N1, N2 <= 256: N <= 65536

// Sizes as 32-bit ints: the host checks that every per-sequence offset fits (L D and N PT below
// 2^31); the batch offsets are formed once per CTA in 64 bits.
struct FftParams {
  int L, D, d_g, l_h;
  int N1, N2;
  int PT;            // signals per sequence: D / 2 (data) or G (spectrum)
  int G;
  int vec;           // q, k, v, y 16-byte aligned and D a multiple of one 16-byte vector
};

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

// exp(-2 pi i num / den) (den a power of two, 0 <= num < den), accurate to a few ulp.
__device__ __forceinline__ float2 twiddle(int num, int den) {
  float s, c;
  sincospif(-2.0f * static_cast<float>(num) / static_cast<float>(den), &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ float2 times_i(float2 a, bool neg) {  // +i a, or -i a when neg
  return neg ? make_float2(a.y, -a.x) : make_float2(-a.y, a.x);
}

// Stockham FFT (self-sorting) of n = 2^k points for kP signals laid out a[point * kP + signal]:
// radix-4 stages while four or more points per sub-transform remain, then one radix-2 stage
// when log2 n is odd.  b is scratch of the same size; tw[k] = W_n^k for k < n.  Forward (W)
// or inverse (W^-1, unscaled).  Returns the buffer holding the result.  All threads take part.
template <bool kInverse>
__device__ float2 *fft_smem(float2 *a, float2 *b, int n, const float2 *tw) {
  for (int ns = 1; ns < n;) {
    const bool r4 = n / ns >= 4;
    const int R = r4 ? 4 : 2;
    const int m = n / R;
    const int step = n / (R * ns);
    for (int e = threadIdx.x; e < m * kP; e += blockDim.x) {
      const int j = e / kP, sig = e % kP;
      const int k = j & (ns - 1);
      const int d = (j - k) * R + k;
      if (r4) {
        float2 w1 = tw[k * step], w2 = tw[2 * k * step], w3 = tw[3 * k * step];
        if (kInverse) {
          w1.y = -w1.y;
          w2.y = -w2.y;
          w3.y = -w3.y;
        }
        const float2 v0 = a[j * kP + sig];
        const float2 v1 = cmul(a[(j + m) * kP + sig], w1);
        const float2 v2 = cmul(a[(j + 2 * m) * kP + sig], w2);
        const float2 v3 = cmul(a[(j + 3 * m) * kP + sig], w3);
        const float2 a0 = make_float2(v0.x + v2.x, v0.y + v2.y);
        const float2 a1 = make_float2(v0.x - v2.x, v0.y - v2.y);
        const float2 b0 = make_float2(v1.x + v3.x, v1.y + v3.y);
        const float2 b1 = times_i(make_float2(v1.x - v3.x, v1.y - v3.y), !kInverse);
        b[d * kP + sig] = make_float2(a0.x + b0.x, a0.y + b0.y);
        b[(d + ns) * kP + sig] = make_float2(a1.x + b1.x, a1.y + b1.y);
        b[(d + 2 * ns) * kP + sig] = make_float2(a0.x - b0.x, a0.y - b0.y);
        b[(d + 3 * ns) * kP + sig] = make_float2(a1.x - b1.x, a1.y - b1.y);
      } else {
        float2 w = tw[k * step];
        if (kInverse) w.y = -w.y;
        const float2 u = a[j * kP + sig];
        const float2 t = cmul(a[(j + m) * kP + sig], w);
        b[d * kP + sig] = make_float2(u.x + t.x, u.y + t.y);
        b[(d + ns) * kP + sig] = make_float2(u.x - t.x, u.y - t.y);
      }
    }
    __syncthreads();
    float2 *x = a;
    a = b;
    b = x;
    ns *= R;
  }
  return a;
}

// tw[k] = W_n^k for k < n; with n2 >= 0 also tw2[k1] = W_N^{n2 k1} for k1 < n (the twiddles
// between the two factors of the four-step transform, for this CTA's n2).
__device__ __forceinline__ void fill_twiddles(float2 *tw, int n, float2 *tw2 = nullptr, int n2 = 0,
                                              int N = 1) {
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    tw[k] = twiddle(k, n);
    if (tw2) tw2[k] = twiddle((n2 * k) & (N - 1), N);
  }
}

// 16-byte vectors of T: 8 / sizeof(T) channel pairs.
template <typename T>
struct PairVec {
  static constexpr int VP = 8 / static_cast<int>(sizeof(T));
  __device__ static void load(const T *p, float (&o)[2 * VP]);
  __device__ static void store(T *p, const float (&o)[2 * VP]);
};
template <>
__device__ inline void PairVec<__nv_bfloat16>::load(const __nv_bfloat16 *p, float (&o)[8]) {
  cc::Vec<__nv_bfloat16>::unpack(cc::Vec<__nv_bfloat16>::load(p), o);
}
template <>
__device__ inline void PairVec<__nv_bfloat16>::store(__nv_bfloat16 *p, const float (&o)[8]) {
  cc::Vec<__nv_bfloat16>::store(p, o);
}
template <>
__device__ inline void PairVec<float>::load(const float *p, float (&o)[4]) {
  cc::Vec<float>::unpack(cc::Vec<float>::load(p), o);
}
template <>
__device__ inline void PairVec<float>::store(float *p, const float (&o)[4]) {
  cc::Vec<float>::store(p, o);
}

// Pass 1.  Block (n2, signal block, b).  Data mode: signal s of sequence b is
// k v at channels 2s, 2s+1 (real, imaginary); spectrum mode: signal s is filter s (real).
// Writes A[b][k1][n2][s] = W_N^{n2 k1} * sum_{n1} z[N2 n1 + n2] W_N1^{n1 k1}.
template <typename T, bool kSpectrum>
__global__ void __launch_bounds__(kThreads)
    fft_pass1_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ h,
                     float2 *__restrict__ A, const FftParams p) {
  extern __shared__ float2 fsm[];
  const int n1len = p.N1;
  float2 *b0 = fsm, *b1 = fsm + n1len * kP, *tw = fsm + 2 * n1len * kP, *tw2 = tw + n1len;
  const int n2 = blockIdx.x;
  const int s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  const int N = p.N1 * p.N2;
  fill_twiddles(tw, n1len, tw2, n2, N);
  if constexpr (kSpectrum) {
    for (int e = threadIdx.x; e < n1len * kP; e += blockDim.x) {
      const int n1 = e / kP, sig = e % kP;
      const int t = p.N2 * n1 + n2, s = s0 + sig;
      b0[e] = make_float2(s < p.PT && t < p.l_h ? __ldg(h + s * p.l_h + t) : 0.f, 0.f);
    }
  } else {
    constexpr int VP = PairVec<T>::VP, NV = kP / VP;
    const T *kb = k + b * p.L * p.D + 2 * s0, *vb = v + b * p.L * p.D + 2 * s0;
    for (int e = threadIdx.x; e < n1len * NV; e += blockDim.x) {
      const int n1 = e / NV, cv = e % NV;
      const int t = p.N2 * n1 + n2, s = s0 + cv * VP;
      float kf[2 * VP], vf[2 * VP];
#pragma unroll
      for (int i = 0; i < 2 * VP; ++i) kf[i] = vf[i] = 0.f;
      if (t < p.L && s < p.PT) {
        const int off = t * p.D + 2 * cv * VP;
        if (p.vec && s + VP <= p.PT) {
          PairVec<T>::load(kb + off, kf);
          PairVec<T>::load(vb + off, vf);
        } else {
          for (int i = 0; i < VP && s + i < p.PT; ++i) {
            kf[2 * i] = cc::to_f32(kb[off + 2 * i]);
            kf[2 * i + 1] = cc::to_f32(kb[off + 2 * i + 1]);
            vf[2 * i] = cc::to_f32(vb[off + 2 * i]);
            vf[2 * i + 1] = cc::to_f32(vb[off + 2 * i + 1]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < VP; ++i)
        b0[n1 * kP + cv * VP + i] = make_float2(kf[2 * i] * vf[2 * i], kf[2 * i + 1] * vf[2 * i + 1]);
    }
  }
  __syncthreads();
  const float2 *r = fft_smem<false>(b0, b1, n1len, tw);
  // A[b][k1][n2][s]: this CTA's signals at k1 lie k1 N2 PT apart
  float2 *ab = A + b * N * p.PT + n2 * p.PT + s0;
  const int kstride = p.N2 * p.PT;
  for (int e = threadIdx.x; e < n1len * kP; e += blockDim.x) {
    const int k1 = e / kP, sig = e % kP;
    if (s0 + sig < p.PT) ab[k1 * kstride + sig] = cmul(r[e], tw2[k1]);
  }
}

// Pass 2.  Block (k1, signal block, b): length-N2 FFT over n2 of A[b][k1][.][s].  Spectrum
// mode writes the spectrum H[k1][k2][g] (signal = group); data mode multiplies by the group's
// H, inverse-transforms over k2 and writes the result back in place.
template <bool kSpectrum>
__global__ void __launch_bounds__(kThreads)
    fft_pass2_kernel(float2 *__restrict__ A, float2 *__restrict__ H, const FftParams p) {
  extern __shared__ float2 fsm[];
  const int n2len = p.N2;
  float2 *b0 = fsm, *b1 = fsm + n2len * kP, *tw = fsm + 2 * n2len * kP;
  const int k1 = blockIdx.x;
  const int s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  fill_twiddles(tw, n2len);
  // A[b][k1][n2][s0 + sig] at row[n2 PT + sig]
  float2 *row = A + (b * p.N1 + k1) * p.N2 * p.PT + s0;
  for (int e = threadIdx.x; e < n2len * kP; e += blockDim.x) {
    const int n2 = e / kP, sig = e % kP;
    b0[e] = s0 + sig < p.PT ? row[n2 * p.PT + sig] : make_float2(0.f, 0.f);
  }
  __syncthreads();
  float2 *r = fft_smem<false>(b0, b1, n2len, tw);
  float2 *o = r == b0 ? b1 : b0;
  const float2 *hk = H + k1 * p.N2 * p.G;  // H[k1][k2][g] at hk[k2 G + g]
  if constexpr (kSpectrum) {
    for (int e = threadIdx.x; e < n2len * kP; e += blockDim.x) {
      const int k2 = e / kP, sig = e % kP;
      if (s0 + sig < p.PT) H[k1 * p.N2 * p.G + k2 * p.G + s0 + sig] = r[e];
    }
  } else {
    for (int e = threadIdx.x; e < n2len * kP; e += blockDim.x) {
      const int k2 = e / kP, sig = e % kP;
      const int s = s0 + sig;
      const int g = s < p.PT ? (2 * s) / p.d_g : 0;
      r[e] = cmul(r[e], hk[k2 * p.G + g]);
    }
    __syncthreads();
    const float2 *y = fft_smem<true>(r, o, n2len, tw);
    for (int e = threadIdx.x; e < n2len * kP; e += blockDim.x) {
      const int n2 = e / kP, sig = e % kP;
      if (s0 + sig < p.PT) row[n2 * p.PT + sig] = y[e];
    }
  }
}

// Pass 3.  Block (n2, signal block, b): W_N^{-n2 k1} times A[b][.][n2][s], inverse length-N1
// FFT over k1, scaled by 1/N: the convolution at t = N2 n1 + n2; y = q * conv for t < L.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    fft_pass3_kernel(const float2 *__restrict__ A, const T *__restrict__ q, T *__restrict__ y,
                     const FftParams p) {
  extern __shared__ float2 fsm[];
  const int n1len = p.N1;
  float2 *b0 = fsm, *b1 = fsm + n1len * kP, *tw = fsm + 2 * n1len * kP, *tw2 = tw + n1len;
  const int n2 = blockIdx.x;
  const int s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  const int N = p.N1 * p.N2;
  fill_twiddles(tw, n1len, tw2, n2, N);
  __syncthreads();
  const float2 *ab = A + b * N * p.PT + n2 * p.PT + s0;
  const int kstride = p.N2 * p.PT;
  for (int e = threadIdx.x; e < n1len * kP; e += blockDim.x) {
    const int k1 = e / kP, sig = e % kP;
    float2 z = make_float2(0.f, 0.f);
    if (s0 + sig < p.PT) {
      const float2 w = tw2[k1];
      z = cmul(ab[k1 * kstride + sig], make_float2(w.x, -w.y));
    }
    b0[e] = z;
  }
  __syncthreads();
  const float2 *r = fft_smem<true>(b0, b1, n1len, tw);
  const float inv = 1.0f / static_cast<float>(N);
  constexpr int VP = PairVec<T>::VP, NV = kP / VP;
  const T *qb = q + b * p.L * p.D + 2 * s0;
  T *yb = y + b * p.L * p.D + 2 * s0;
  for (int e = threadIdx.x; e < n1len * NV; e += blockDim.x) {
    const int n1 = e / NV, cv = e % NV;
    const int t = p.N2 * n1 + n2, s = s0 + cv * VP;
    if (t >= p.L || s >= p.PT) continue;
    const int off = t * p.D + 2 * cv * VP;
    const float2 *rr = r + n1 * kP + cv * VP;
    if (p.vec && s + VP <= p.PT) {
      float qf[2 * VP], o[2 * VP];
      PairVec<T>::load(qb + off, qf);
#pragma unroll
      for (int i = 0; i < VP; ++i) {
        o[2 * i] = qf[2 * i] * (rr[i].x * inv);
        o[2 * i + 1] = qf[2 * i + 1] * (rr[i].y * inv);
      }
      PairVec<T>::store(yb + off, o);
    } else {
      for (int i = 0; i < VP && s + i < p.PT; ++i) {
        cc::from_f32(cc::to_f32(qb[off + 2 * i]) * (rr[i].x * inv), yb + off + 2 * i);
        cc::from_f32(cc::to_f32(qb[off + 2 * i + 1]) * (rr[i].y * inv), yb + off + 2 * i + 1);
      }
    }
  }
}

}  // namespace fft
}  // namespace hyena
