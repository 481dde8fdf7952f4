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
//  * fir_tiled_kernel: the direct sum for any supported shape and alignment, tiled through
//    shared memory (also the backward's transposed product).  The fallback for shapes the
//    fast kernels do not cover.
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

// Programmatic dependent launch, for kernels launched with programmatic stream serialisation:
// let the next kernel of the stream be scheduled at once, then wait until the previous one has
// completed and its writes are visible.  Call before the first global-memory access.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

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
  pdl_enter();  // launched with programmatic stream serialisation
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

// Tiled direct sum, any shape.  A CTA takes 64 channels x 128 rows of one sequence; thread
// (channel tid % 64, row group tid / 64) owns rows 32 rg .. 32 rg + 31 of its channel as four
// blocks of 8.  Taps go in chunks of 128: the chunk's source rows (255 x 64, fp32) are staged in
// shared memory, then every thread slides four 8-row register windows along them, one shared
// load per 8 FMAs.  Each output sums its taps in the order j = 0, 1, ... (fmaf from 0): taps
// that reach rows with no data add exact zeros, so the results are those of a plain per-output
// loop.
//   kAnti = false: y[t] = q[t] sum_j h[j] x[t - j], x = k v (rows -Lh .. -1 from the history
//                  k_hist, v_hist, zero before them);
//   kAnti = true:  dx[t] = sum_j h[j] dz[t + j], dz = q dy (zero from L on); writes
//                  dk = dx v and dv = dx k (the backward's transposed product).
constexpr int kTileC = 64, kTileR = 128, kTileJ = 128, kTileThreads = 256;
constexpr int kTileWin = kTileR + kTileJ - 1;
constexpr int kTileSmemBytes = kTileWin * kTileC * 4;

template <typename T, bool kAnti>
__global__ void __launch_bounds__(kTileThreads)
    fir_tiled_kernel(const T *__restrict__ a0, const T *__restrict__ a1,
                     const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ h, T *__restrict__ o0, T *__restrict__ o1,
                     long long B, long long L, long long D, int d_g, int l_h,
                     const T *__restrict__ kh, const T *__restrict__ vh, long long Lh,
                     const unsigned *__restrict__ run_if, unsigned run_token) {
  // forward: a0 = q, a1 unused, o0 = y;  anti: a0 = q, a1 = dy, o0 = dk, o1 = dv.
  // run_if (anti only; may be null): a device word; unless it holds run_token the kernel does
  // nothing (the fp32 recomputation behind the tensor-core backward, needed only where that
  // kernel raised its flag).  Such a launch may start early (programmatic dependent launch): it
  // waits for the previous kernels of the stream before it reads anything.
  if constexpr (kAnti) {
    if (run_if) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      if (*run_if != run_token) return;
    }
  }
  extern __shared__ float xs[];  // [kTileWin][kTileC]
  const int cl = threadIdx.x % kTileC, rg = threadIdx.x / kTileC;
  const long long n_ct = (D + kTileC - 1) / kTileC, n_rt = (L + kTileR - 1) / kTileR;
  const long long n_tiles = B * n_rt * n_ct;
  // tiles (channel tile fastest, then row tile, then sequence), grid-stride over the CTAs
  for (long long tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
  const long long c0 = (tile % n_ct) * kTileC;
  const long long t0 = ((tile / n_ct) % n_rt) * kTileR;
  const long long b = tile / (n_ct * n_rt);
  const long long c = c0 + cl;
  const bool live_c = c < D;
  const float *hg = h + (live_c ? c / d_g : 0) * l_h;
  const long long seq = b * L * D;
  float acc[4][8];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[q4][i] = 0.f;

  for (int j0 = 0; j0 < l_h; j0 += kTileJ) {
    // source row of window row w: base + w
    const long long base = kAnti ? t0 + j0 : t0 - j0 - (kTileJ - 1);
    __syncthreads();  // the previous chunk's window has been read
    for (int e = threadIdx.x; e < kTileWin * kTileC; e += kTileThreads) {
      const int w = e / kTileC, ce = e % kTileC;
      const long long sr = base + w, gc = c0 + ce;
      float val = 0.f;
      if (gc < D) {
        if (sr >= 0 && sr < L) {
          const long long a = seq + sr * D + gc;
          val = kAnti ? to_f32(a0[a]) * to_f32(a1[a]) : to_f32(k[a]) * to_f32(v[a]);
        } else if (!kAnti && sr < 0 && sr >= -Lh) {
          const long long a = (b * Lh + Lh + sr) * D + gc;
          val = to_f32(kh[a]) * to_f32(vh[a]);
        }
      }
      xs[w * kTileC + ce] = val;
    }
    __syncthreads();
    const int nj = min(kTileJ, l_h - j0);
    // taps in groups of 8 (past l_h: h = 0, which adds exact zeros): an 8 x 8 block of a row
    // block's outputs and the group's taps reads 15 window rows, u = i - t + 7 (forward) or
    // u = i + t (anti) for output i and tap t of the group
    for (int jj0 = 0; jj0 < nj; jj0 += 8) {
      float hv[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) hv[t] = jj0 + t < nj ? __ldg(hg + j0 + jj0 + t) : 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r0 = rg * 32 + q4 * 8;
        const int w0 = kAnti ? r0 + jj0 : r0 + kTileJ - 8 - jj0;
        float xw[15];
#pragma unroll
        for (int u = 0; u < 15; ++u) xw[u] = xs[(w0 + u) * kTileC + cl];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[q4][i] = fmaf(hv[t], xw[kAnti ? i + t : i - t + 7], acc[q4][i]);
      }
    }
  }
  if (live_c) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const long long t = t0 + rg * 32 + q4 * 8 + i;
        if (t >= L) continue;
        const long long a = seq + t * D + c;
        if (kAnti) {
          from_f32(acc[q4][i] * to_f32(v[a]), o0 + a);
          from_f32(acc[q4][i] * to_f32(k[a]), o1 + a);
        } else {
          from_f32(to_f32(a0[a]) * acc[q4][i], o0 + a);
        }
      }
    }
  }
  }  // tiles
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
