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
// Each length-n transform (n = R1 R2, both at most 16) runs as in-register DFTs joined by one
// exchange through shared memory: a thread holds R1 points of one signal (stride R2), transforms
// them, applies W_n^{j k1} and stores them; then the R2 points of each k1 are shared by
// P = 16 / R1 threads, each taking the first radix-P step over all of them on the way out of
// shared memory and an (R2 / P)-point DFT in registers, so that every thread works in both
// halves and holds at most max(R1, R2 / P) values.  16 signals (channel pairs) per CTA, 16
// threads per signal.  Twiddles come from sincospif, tabled once per CTA.  The intermediate spectra live in a caller-owned fp32
// workspace laid out [b][k1][n2][pair]: every pass moves 16 contiguous complex values (128
// bytes) per index.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "fir_cuda_core.cuh"

namespace hyena {
namespace fft {

constexpr int kP = 16;          // signals (channel pairs) per CTA
constexpr int kThreads = 256;   // 16 threads per signal
constexpr int kMinLen = 16, kMaxLen = 256;  // N1, N2 in [16, 256]: N in [256, 65536]

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
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }

// exp(-2 pi i num / den) (den a power of two, 0 <= num < den), accurate to a few ulp.
__device__ __forceinline__ float2 twiddle(int num, int den) {
  float s, c;
  sincospif(-2.0f * static_cast<float>(num) / static_cast<float>(den), &s, &c);
  return make_float2(c, s);
}

// d * W_16^w (or its conjugate) for a compile-time w < 8; W_16^w = cos(pi w / 8) - i sin(pi w / 8).
template <int w, bool kInv>
__device__ __forceinline__ float2 w16mul(float2 d) {
  constexpr float c8 = 0.92387953251128674f, s8 = 0.38268343236508978f, r2 = 0.70710678118654752f;
  constexpr float cs[8] = {1.f, c8, r2, s8, 0.f, -s8, -r2, -c8};
  constexpr float sn[8] = {0.f, s8, r2, c8, 1.f, c8, r2, s8};  // sin(pi w / 8) >= 0
  if constexpr (w == 0) {
    return d;
  } else if constexpr (w == 4) {  // -i (forward) or +i (inverse)
    return kInv ? make_float2(-d.y, d.x) : make_float2(d.y, -d.x);
  } else {
    const float c = cs[w], s = kInv ? sn[w] : -sn[w];
    return make_float2(d.x * c - d.y * s, d.x * s + d.y * c);
  }
}

__host__ __device__ constexpr int brev(int i, int bits) {
  int r = 0;
  for (int b = 0; b < bits; ++b) r |= ((i >> b) & 1) << (bits - 1 - b);
  return r;
}
__host__ __device__ constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n / 2); }

// t[bit-reverse(i)] = v[i] for every i, with compile-time indices.
template <int R, int i = 0>
__device__ __forceinline__ void brev_copy(float2 (&t)[R], const float2 (&v)[R]) {
  if constexpr (i < R) {
    t[brev(i, ilog2(R))] = v[i];
    brev_copy<R, i + 1>(t, v);
  }
}

// One radix-2 decimation-in-frequency stage of span h over R registers.
template <int R, int h, bool kInv, int i = 0, int j = 0>
__device__ __forceinline__ void dif_stage(float2 (&v)[R]) {
  if constexpr (i < R) {
    if constexpr (j < h) {
      const float2 a = v[i + j], b = v[i + j + h];
      v[i + j] = make_float2(a.x + b.x, a.y + b.y);
      v[i + j + h] = w16mul<j * (16 / (2 * h)), kInv>(make_float2(a.x - b.x, a.y - b.y));
      dif_stage<R, h, kInv, i, j + 1>(v);
    } else {
      dif_stage<R, h, kInv, i + 2 * h, 0>(v);
    }
  }
}

template <int R, int h, bool kInv>
__device__ __forceinline__ void dif_all(float2 (&v)[R]) {
  if constexpr (h >= 1) {
    dif_stage<R, h, kInv>(v);
    dif_all<R, h / 2, kInv>(v);
  }
}

// In-register DFT of R (2..16) points, natural order in and out, forward or inverse (unscaled).
template <int R, bool kInv>
__device__ __forceinline__ void dft_reg(float2 (&v)[R]) {
  dif_all<R, R / 2, kInv>(v);
  float2 t[R];
  brev_copy<R>(t, v);
#pragma unroll
  for (int i = 0; i < R; ++i) v[i] = t[i];
}

// The split n = R1 R2 of a transform length (R1, R2 <= 16).
template <int n> struct Split;
template <> struct Split<16> { static constexpr int R1 = 4, R2 = 4; };
template <> struct Split<32> { static constexpr int R1 = 4, R2 = 8; };
template <> struct Split<64> { static constexpr int R1 = 8, R2 = 8; };
template <> struct Split<128> { static constexpr int R1 = 8, R2 = 16; };
template <> struct Split<256> { static constexpr int R1 = 16, R2 = 16; };

// z * W_4^e (e in 0..3; W_4 = -i), or its conjugate, for a run-time e.
template <bool kInv>
__device__ __forceinline__ float2 w4mul(float2 z, int e) {
  if (e & 2) z = make_float2(-z.x, -z.y);
  if (e & 1) z = kInv ? make_float2(-z.y, z.x) : make_float2(z.y, -z.x);
  return z;
}

// Length-n transforms of 16 signals by the CTA, 16 threads per signal (sig = thread % 16,
// idx = thread / 16).  n = R1 R2; the R2-point half is shared by P = 16 / R1 threads per k1,
// each computing M = R2 / P of its outputs, so that all 16 threads hold values in both halves.
// Layouts (per signal):
//   "A" layout: thread idx = j < R2 holds x[j + R2 m], m < R1   (natural time order)
//   "B" layout: thread idx = P k1 + q holds X[k1 + R1 (P r + q)], r < M  (see bfreq)
// ex is n x 16 complex of shared memory, tw[k] = W_n^k.  Both functions end with the result
// in registers; they synchronise the CTA around their use of ex.
template <int n>
struct BLay {
  static constexpr int R1 = Split<n>::R1, R2 = Split<n>::R2;
  static constexpr int P = 16 / R1, M = R2 / P;
  static_assert(P * R1 == 16 && M * P == R2, "split of the R2-point half");
};

// Frequency index held in register r of B-layout thread idx.
template <int n>
__device__ __forceinline__ int bfreq(int idx, int r) {
  using BL = BLay<n>;
  return idx / BL::P + BL::R1 * (BL::P * r + idx % BL::P);
}

// A -> B: R1-point DFTs, twiddles W_n^{j k1}, exchange, then the R2-point DFT over j split
// four-step style: X[k1 + R1 (P r + q)] = sum_{j < M} W_M^{j r} W_R2^{j q}
// sum_{p < P} W_P^{p q} y_k1[j + p M].
template <int n, bool kInv>
__device__ __forceinline__ void a_to_b(float2 (&va)[Split<n>::R1], float2 (&vb)[BLay<n>::M],
                                       float2 *ex, const float2 *tw, int idx, int sig) {
  using BL = BLay<n>;
  constexpr int R1 = BL::R1, R2 = BL::R2, P = BL::P, M = BL::M;
  __syncthreads();  // ex is free
  if (idx < R2) {
    dft_reg<R1, kInv>(va);
#pragma unroll
    for (int k1 = 0; k1 < R1; ++k1) {
      const float2 w = tw[(idx * k1) & (n - 1)];
      ex[(k1 * R2 + idx) * kP + sig] = cmul(va[k1], kInv ? cconj(w) : w);
    }
  }
  __syncthreads();
  const int k1 = idx / P, q = idx % P;
#pragma unroll
  for (int j = 0; j < M; ++j) {
    float2 z = ex[(k1 * R2 + j) * kP + sig];
#pragma unroll
    for (int p = 1; p < P; ++p) {
      const float2 t = w4mul<kInv>(ex[(k1 * R2 + j + p * M) * kP + sig], ((4 / P) * p * q) & 3);
      z = make_float2(z.x + t.x, z.y + t.y);
    }
    if (P > 1 && j > 0) {
      const float2 w = tw[(R1 * j * q) & (n - 1)];
      z = cmul(z, kInv ? cconj(w) : w);
    }
    vb[j] = z;
  }
  dft_reg<M, kInv>(vb);
}

// B -> A, the mirror of a_to_b: M-point DFTs, W_R2^{j q}, exchange, the P-point combination
// and W_n^{k1 j'} (j' = j + p M), then R1-point DFTs.
template <int n, bool kInv>
__device__ __forceinline__ void b_to_a(float2 (&vb)[BLay<n>::M], float2 (&va)[Split<n>::R1],
                                       float2 *ex, const float2 *tw, int idx, int sig) {
  using BL = BLay<n>;
  constexpr int R1 = BL::R1, R2 = BL::R2, P = BL::P, M = BL::M;
  __syncthreads();
  const int k1 = idx / P, q = idx % P;
  dft_reg<M, kInv>(vb);
#pragma unroll
  for (int j = 0; j < M; ++j) {
    float2 z = vb[j];
    if (P > 1 && j > 0) {
      const float2 w = tw[(R1 * j * q) & (n - 1)];
      z = cmul(z, kInv ? cconj(w) : w);
    }
    ex[((k1 * P + q) * M + j) * kP + sig] = z;
  }
  __syncthreads();
  if (idx < R2) {
    const int j = idx % M, p = idx / M;
#pragma unroll
    for (int kk = 0; kk < R1; ++kk) {
      float2 z = ex[((kk * P) * M + j) * kP + sig];
#pragma unroll
      for (int qq = 1; qq < P; ++qq) {
        const float2 t = w4mul<kInv>(ex[((kk * P + qq) * M + j) * kP + sig], ((4 / P) * p * qq) & 3);
        z = make_float2(z.x + t.x, z.y + t.y);
      }
      const float2 w = tw[(idx * kk) & (n - 1)];
      va[kk] = cmul(z, kInv ? cconj(w) : w);
    }
    dft_reg<R1, kInv>(va);
  }
}

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

// Pass 1.  Block (n2, signal block, b): signal s of sequence b is k v at channels 2s, 2s+1
// (real, imaginary) -- or, in spectrum mode, filter s (real).  Writes
// A[b][k][n2][s] = W_N^{n2 k} * sum_{n1} z[N2 n1 + n2] W_N1^{n1 k}, k < N1.
template <typename T, bool kSpectrum, int N1>
__global__ void __launch_bounds__(kThreads)
    fft_pass1_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ h,
                     float2 *__restrict__ A, const FftParams p) {
  constexpr int R1 = Split<N1>::R1, R2 = Split<N1>::R2;
  __shared__ float2 ex[N1 * kP];
  __shared__ float2 tw[N1], tw2[N1];
  const int n2 = blockIdx.x, s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  const int N = N1 * p.N2;
  const int idx = threadIdx.x / kP, sig = threadIdx.x % kP;
  fill_twiddles(tw, N1, tw2, n2, N);
  cc::pdl_enter();  // launched with programmatic stream serialisation (the tables overlap)
  // stage the rows t = N2 n1 + n2 of the CTA's 16 signals: ex[n1 * 16 + signal]
  if constexpr (kSpectrum) {
    for (int e = threadIdx.x; e < N1 * kP; e += blockDim.x) {
      const int n1 = e / kP, sg = e % kP;
      const int t = p.N2 * n1 + n2, s = s0 + sg;
      ex[e] = make_float2(s < p.PT && t < p.l_h ? __ldg(h + s * p.l_h + t) : 0.f, 0.f);
    }
  } else {
    constexpr int VP = PairVec<T>::VP, NV = kP / VP;
    const T *kb = k + b * p.L * p.D + 2 * s0, *vb = v + b * p.L * p.D + 2 * s0;
    for (int e = threadIdx.x; e < N1 * NV; e += blockDim.x) {
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
        ex[n1 * kP + cv * VP + i] = make_float2(kf[2 * i] * vf[2 * i], kf[2 * i + 1] * vf[2 * i + 1]);
    }
  }
  __syncthreads();
  float2 va[R1], vb[BLay<N1>::M];
  if (idx < R2) {
#pragma unroll
    for (int m = 0; m < R1; ++m) va[m] = ex[(idx + R2 * m) * kP + sig];
  }
  a_to_b<N1, false>(va, vb, ex, tw, idx, sig);
  if (s0 + sig < p.PT) {
    float2 *ab = A + b * N * p.PT + n2 * p.PT + s0 + sig;
    const int kstride = p.N2 * p.PT;
#pragma unroll
    for (int r = 0; r < BLay<N1>::M; ++r) {
      const int kk = bfreq<N1>(idx, r);
      ab[kk * kstride] = cmul(vb[r], tw2[kk]);
    }
  }
}

// Pass 2.  Block (k1, signal block, b): length-N2 transform over n2 of A[b][k1][.][s].  Spectrum
// mode writes the spectrum H[k1][k2][g] (signal = group); data mode multiplies by the group's
// H, transforms back and writes the result in place.
template <bool kSpectrum, int N2>
__global__ void __launch_bounds__(kThreads, N2 <= 128 ? 8 : (kSpectrum ? 1 : 4))
    fft_pass2_kernel(float2 *__restrict__ A, float2 *__restrict__ H, const FftParams p) {
  constexpr int R1 = Split<N2>::R1, R2 = Split<N2>::R2;
  constexpr int M = BLay<N2>::M;
  __shared__ float2 ex[N2 * kP];
  __shared__ float2 tw[N2];
  const int k1 = blockIdx.x, s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  const int idx = threadIdx.x / kP, sig = threadIdx.x % kP;
  const bool live = s0 + sig < p.PT;
  fill_twiddles(tw, N2);
  cc::pdl_enter();  // launched with programmatic stream serialisation (the table overlaps)
  // A[b][k1][n2][s0 + sig] at row[n2 PT]
  float2 *row = A + (b * p.N1 + k1) * N2 * p.PT + s0 + sig;
  float2 va[R1], vb[BLay<N2>::M];
  if (idx < R2) {
#pragma unroll
    for (int m = 0; m < R1; ++m)
      va[m] = live ? row[(idx + R2 * m) * p.PT] : make_float2(0.f, 0.f);
  }
  a_to_b<N2, false>(va, vb, ex, tw, idx, sig);  // synchronises before using ex (tw is filled)
  if constexpr (kSpectrum) {
    if (live) {
#pragma unroll
      for (int r = 0; r < BLay<N2>::M; ++r)
        H[(k1 * N2 + bfreq<N2>(idx, r)) * p.G + s0 + sig] = vb[r];
    }
  } else {
    // the group's filter spectrum at this thread's frequencies (L2-resident)
    const float2 *hk = H + k1 * N2 * p.G + (live ? (2 * (s0 + sig)) / p.d_g : 0);
#pragma unroll
    for (int r = 0; r < M; ++r) vb[r] = cmul(vb[r], hk[bfreq<N2>(idx, r) * p.G]);
    b_to_a<N2, true>(vb, va, ex, tw, idx, sig);
    if (idx < R2 && live) {
#pragma unroll
      for (int m = 0; m < R1; ++m) row[(idx + R2 * m) * p.PT] = va[m];
    }
  }
}

// Pass 3.  Block (n2, signal block, b): W_N^{-n2 k} times A[b][k][n2][s], inverse length-N1
// transform over k, scaled by 1/N: the convolution at t = N2 n1 + n2; y = q * conv for t < L.
template <typename T, int N1>
__global__ void __launch_bounds__(kThreads)
    fft_pass3_kernel(const float2 *__restrict__ A, const T *__restrict__ q, T *__restrict__ y,
                     const FftParams p) {
  constexpr int R1 = Split<N1>::R1, R2 = Split<N1>::R2;
  __shared__ float2 ex[N1 * kP];
  __shared__ float2 tw[N1], tw2[N1];
  const int n2 = blockIdx.x, s0 = blockIdx.y * kP;
  const long long b = blockIdx.z;
  const int N = N1 * p.N2;
  const int idx = threadIdx.x / kP, sig = threadIdx.x % kP;
  fill_twiddles(tw, N1, tw2, n2, N);
  cc::pdl_enter();  // launched with programmatic stream serialisation (the tables overlap)
  __syncthreads();
  float2 va[R1], vb[BLay<N1>::M];
  {
    const bool live = s0 + sig < p.PT;
    const float2 *ab = A + b * N * p.PT + n2 * p.PT + s0 + sig;
    const int kstride = p.N2 * p.PT;
#pragma unroll
    for (int r = 0; r < BLay<N1>::M; ++r) {
      const int kk = bfreq<N1>(idx, r);
      vb[r] = live ? cmul(ab[kk * kstride], cconj(tw2[kk])) : make_float2(0.f, 0.f);
    }
  }
  b_to_a<N1, true>(vb, va, ex, tw, idx, sig);
  // x[n1 = idx + R2 m] * N1 N2 in va: through ex to rows of 16 signals
  __syncthreads();
  if (idx < R2) {
#pragma unroll
    for (int m = 0; m < R1; ++m) ex[(idx + R2 * m) * kP + sig] = va[m];
  }
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(N);
  constexpr int VP = PairVec<T>::VP, NV = kP / VP;
  const T *qb = q + b * p.L * p.D + 2 * s0;
  T *yb = y + b * p.L * p.D + 2 * s0;
  for (int e = threadIdx.x; e < N1 * NV; e += blockDim.x) {
    const int n1 = e / NV, cv = e % NV;
    const int t = p.N2 * n1 + n2, s = s0 + cv * VP;
    if (t >= p.L || s >= p.PT) continue;
    const int off = t * p.D + 2 * cv * VP;
    const float2 *rr = ex + n1 * kP + cv * VP;
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
