/*
 * hyena_conv.h -- C ABI of the B200 (sm_100a) gated, grouped, depthwise causal FIR.
 *
 * Operation (Hyena-SE / Hyena-MR operators of StripedHyena 2; the convolution is the causal FIR
 * sum of the page "04. Hardware-aware convolution kernels", Sec. 1, gated by q and by k):
 *
 *     y[b,t,c] = q[b,t,c] * sum_{j=0}^{min(l_h-1, t)} h[c / d_g][j] * k[b,t-j,c] * v[b,t-j,c]
 *
 * computed with the block-Toeplitz method of the same page (Sec. 2 block convolution, Sec. 3
 * two-stage form Yhat_n = H0 Xhat_n + H1 Xhat_{n-1}, Xhat_{-1} = 0).
 *
 * Conventions shared by every entry point:
 *   - q, k, v, y are DEVICE pointers to [B, L, D] row-major tensors (channels contiguous),
 *     except in hyena_conv_fwd_from_host, which takes HOST buffers.
 *   - h is a DEVICE pointer to fp32 [D / d_g, l_h], natural tap order: h[g][0] multiplies the
 *     current token.  Channel c belongs to group c / d_g (contiguous groups).
 *   - Every sequence b starts from zero history; no state is kept between calls.
 *   - The caller owns every buffer.  The library allocates no device memory in these calls.
 *     Each call is asynchronous on `stream` (NULL = the legacy default stream) and returns as
 *     soon as the work is queued.
 *   - y must not overlap q, k or v.
 *   - B == 0 or L == 0 is an empty problem: nothing is launched and HYENA_OK is returned.
 *   - Return value: HYENA_OK or one of the HYENA_ERR_* codes below.  Argument errors are
 *     detected on the host before anything is queued.  HYENA_ERR_CUDA reports a launch
 *     failure (cudaGetLastError).  Events inside a running kernel (a bounded wait that ran
 *     out; a tile recomputed in fp32 because an fp16 operand left its range) are recorded in
 *     a per-device status word that hyena_device_status() reads.
 *   - The library keeps per-device state from the first call on each device (kernel
 *     attributes, the host-buffer pipeline's streams, the address of the fixed scratch of
 *     hyena_conv_bwd_static_scratch).  cudaDeviceReset destroys what it refers to: do not call
 *     the library on a device after resetting it in the same process.
 */
#ifndef HYENA_CONV_H
#define HYENA_CONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t (an opaque driver stream handle). */
typedef struct CUstream_st *cudaStream_t;

enum hyena_status {
    HYENA_OK = 0,
    HYENA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, D % d_g != 0, l_h < 1,
                                    l_b < 1, overlapping y, unknown dtype/algo */
    HYENA_ERR_UNSUPPORTED = 2,   /* a forced algorithm cannot run this shape or alignment */
    HYENA_ERR_MISALIGNED = 3,    /* a pointer is not aligned to its element size */
    HYENA_ERR_CUDA = 4           /* the CUDA runtime reported an error for this call */
};

enum hyena_dtype {
    HYENA_DTYPE_BF16 = 0,        /* q, k, v, y bf16; fp32 accumulation */
    HYENA_DTYPE_F32 = 1          /* q, k, v, y fp32; fp32 accumulation */
};

enum hyena_algo {
    HYENA_ALGO_AUTO = 0,         /* pick the fastest algorithm that supports the problem */
    HYENA_ALGO_TENSOR = 1,       /* tcgen05 tensor-core block-Toeplitz GEMM (bf16 only;
                                    D % 64 == 0, d_g in {16, 32, 64}; l_h <= 641 for
                                    d_g == 64, <= 257 for d_g == 32, <= 65 for d_g == 16;
                                    16-byte aligned tensors) */
    HYENA_ALGO_WINDOW = 2,       /* CUDA-core register sliding window, forward and backward
                                    (l_h <= 16; d_g a multiple of 8 channels for bf16, 4 for
                                    fp32; 16-byte aligned tensors) */
    HYENA_ALGO_DIRECT = 3,       /* CUDA-core direct sum, tiled through shared memory; any
                                    supported shape */
    HYENA_ALGO_FFT = 4           /* forward only: single-pass block FFT (overlap-save) on the
                                    CUDA cores in fp32, no workspace; l_h <= 8192 for bf16,
                                    <= 4096 for fp32; d_g a multiple of 2P channels for the
                                    transform length N chosen (bf16: P = 8, 4, 2, 1 channel
                                    pairs at N = 1024, 2048, 4096, 8192; fp32: P = 4, 2, 1 at
                                    N = 1024, 2048, 4096); tensors aligned to the 2P-channel
                                    row piece (at most 16 bytes) */
};

/* Bits of the per-device status word (hyena_device_status). */
enum hyena_device_status_bits {
    HYENA_DEVICE_TIMEOUT = 1u,      /* a bounded wait inside a kernel gave up; output invalid */
    HYENA_DEVICE_F16_RANGE = 2u     /* information, not an error: in the tensor-core forward
                                       an fp16 operand left its range even after the kernel's
                                       power-of-two scaling (a scaled |k*v| above 65504, or a
                                       warp's rows all far below the sequence run's first
                                       tile), and the tiles reading it were recomputed in fp32
                                       on the CUDA cores; in the tensor-core backward an fp16
                                       operand exceeded 65504 (or a group's taps all lay below
                                       2^-10) and dk, dv, dh were recomputed in fp32; outputs
                                       are valid */
};

/*
 * Gated grouped causal FIR forward, bf16 q/k/v/y (the Hyena-SE / Hyena-MR operator).
 * l_b is the block size of the block-Toeplitz decomposition (page 04, Sec. 2).  Any l_h >= 1 is
 * accepted: the block form with S = 1 + ceil((l_h - 1) / l_b) sub-block diagonals is exact for
 * every filter length (the two-stage form of Sec. 3 is the case S = 2, l_h <= l_b + 1), so the
 * result does not depend on l_b.  The kernels pick their own internal block size.  Filters
 * of 17 taps or more that the tensor path does not take (longer than its limit, fp32, or
 * d_g outside {16, 32, 64}) run on the single-pass block FFT (HYENA_ALGO_FFT) where it
 * applies, else on the CUDA-core direct sum; hyena_conv_fwd_fft (with a workspace) takes
 * filters of any length.  All tensors 2-byte aligned.
 * Precision: on the tensor-core path the MMA operands are fp16 (x = k v formed exactly in
 * fp32; h), each scaled by a power of two first (per group for h, per sequence run for x),
 * with fp32 accumulation; tiles whose scaled operands still leave fp16's range are recomputed
 * in fp32 on the CUDA cores (HYENA_DEVICE_F16_RANGE).  The CUDA-core paths are fp32.  y is
 * rounded once to bf16.
 */
int hyena_conv_fwd(const void *q, const void *k, const void *v, const float *h, void *y,
                   int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                   cudaStream_t stream);

/* The same operation with fp32 q/k/v/y (4-byte aligned). */
int hyena_conv_fwd_f32(const float *q, const float *k, const float *v, const float *h,
                       float *y, int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                       cudaStream_t stream);

/*
 * The same operation with the element type (enum hyena_dtype) and the algorithm
 * (enum hyena_algo) chosen by the caller.  A forced algorithm that cannot run the problem
 * returns HYENA_ERR_UNSUPPORTED without queuing anything.
 */
int hyena_conv_fwd_ex(const void *q, const void *k, const void *v, const float *h, void *y,
                      int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                      int dtype, int algo, cudaStream_t stream);

/*
 * One shard of longer sequences: the same operation as hyena_conv_fwd_ex over rows 0 .. L-1
 * of every sequence, where the L_hist rows that precede row 0 are given instead of zero
 * history (page 04, Sec. 3: output chunk n needs input chunk n-1; page 01, Sec. 5 names
 * point-to-point context parallelism, which cuts a sequence across devices):
 *
 *     y[b,t,c] = q[b,t,c] * sum_{j=0}^{min(l_h-1, t+L_hist)} h[c/d_g][j] * x(b, t-j, c),
 *     x(b, s, c) = k[b,s,c] v[b,s,c] for s >= 0,
 *                  k_hist[b, L_hist+s, c] v_hist[b, L_hist+s, c] for s < 0.
 *
 * k_hist, v_hist: DEVICE [B, L_hist, D] tensors of `dtype` (row L_hist-1 immediately precedes
 * row 0); only their last min(L_hist, l_h-1) rows are read.  L_hist == 0 is zero history
 * (k_hist, v_hist may then be NULL) and gives exactly hyena_conv_fwd_ex.  The history must not
 * overlap y.  Every algorithm takes history; HYENA_ALGO_TENSOR and HYENA_ALGO_WINDOW also need
 * k_hist and v_hist 16-byte aligned.  Errors: as hyena_conv_fwd_ex, plus HYENA_ERR_INVALID_ARG
 * for L_hist < 0, NULL history with L_hist > 0 or history that overlaps y, and
 * HYENA_ERR_MISALIGNED for history not aligned to its element size.
 */
int hyena_conv_fwd_hist(const void *q, const void *k, const void *v, const float *h, void *y,
                        const void *k_hist, const void *v_hist, int64_t L_hist, int64_t B,
                        int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype, int algo,
                        cudaStream_t stream);

/*
 * Host-only: bytes of device workspace hyena_conv_fwd_fft needs for this shape (a multiple of
 * 256), minus HYENA_ERR_INVALID_ARG for a bad shape, or minus HYENA_ERR_UNSUPPORTED where the
 * FFT path does not apply (odd D or d_g, or L + l_h - 1 > 65536).  Touches no device.  The
 * workspace holds the fp32 spectra: 4 B L_fft D bytes for the data plus 16 L_fft D / d_g for
 * the filters, L_fft the power of two >= max(256, L + l_h - 1) (256 MiB of data spectra at
 * B = 1, L = l_h = 8192, D = 4096).
 */
int64_t hyena_conv_fwd_fft_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h);

/*
 * The same operation as hyena_conv_fwd_ex, evaluated by FFT: the convolution of every channel
 * with its group's filter as a cyclic convolution of length L_fft (zero-padded, so exact for
 * t < L), computed with a four-step FFT in three passes over the workspace.  For long filters
 * (the Hyena-LI operator of StripedHyena 2, overview page, Sec. 3 operator table: long
 * implicit filters, FFT convolution; the direct and block-Toeplitz forms cost O(L l_h) per
 * channel, this one O(L log L)).  Any l_h >= 1; needs D and d_g even (two channels of a group
 * share one complex transform) and L + l_h - 1 <= 65536.  dtype bf16 or fp32 (q, k, v, y);
 * the transforms run in fp32.
 * workspace: DEVICE scratch of at least hyena_conv_fwd_fft_workspace_bytes() bytes, 16-byte
 * aligned, owned by the caller, unused after the queued work ends.
 * Errors: as hyena_conv_fwd_ex, plus HYENA_ERR_UNSUPPORTED as above, HYENA_ERR_INVALID_ARG for
 * a NULL or too small workspace, HYENA_ERR_MISALIGNED for a misaligned one.
 */
int hyena_conv_fwd_fft(const void *q, const void *k, const void *v, const float *h, void *y,
                       int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Host-only: bytes of device workspace hyena_conv_fwd_from_host needs (a multiple of 256), or
 * minus HYENA_ERR_INVALID_ARG for a bad shape, dtype or chunk < 1.  Touches no device.  The
 * workspace holds three chunk slots of q, k, v and y, (min(L, chunk) + l_h - 1) rows of D
 * elements each, and the filters: 12 (min(L, chunk) + l_h - 1) D elem + 4 (D / d_g) l_h
 * bytes, each buffer rounded up to 256 bytes.
 */
int64_t hyena_conv_fwd_from_host_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g,
                                                 int l_h, int dtype, int64_t chunk);

/*
 * The forward of hyena_conv_fwd_ex (AUTO) with q, k, v, h and y in HOST memory: the
 * end-to-end call, host-to-device copies, kernels and device-to-host copies queued by the
 * library.  Each sequence is processed in chunks of `chunk` rows: rows [t0, t1) of q, k, v
 * travel to the device once, the l_h - 1 rows of k and v before them (page 04, Sec. 3: output
 * chunk n needs only input chunk n-1) are copied on the device from the previous chunk, the
 * block is computed as a sequence of its own, which gives exactly the whole sequence's rows
 * t0 .. t1-1, and those rows come back into y.  Three chunk slots of the workspace rotate
 * over three library streams (copy in, compute, copy out) so that the copies in both
 * directions overlap the kernels; with page-locked (pinned) host buffers every copy is
 * asynchronous, with pageable ones the copies still complete correctly but may serialise.
 *
 * q, k, v, y: HOST [B, L, D] of `dtype`; h: HOST [D / d_g, l_h] fp32.  workspace: DEVICE,
 * 256-byte aligned, at least hyena_conv_fwd_from_host_workspace_bytes() bytes, owned by the
 * caller.  The call is ordered after the work already queued on `stream`, and `stream` waits
 * for its last copy: synchronise `stream` before reading y, and keep the host buffers and the
 * workspace alive until then.  The library's streams and events are created once per device;
 * calls on one device are serialised on the host.  Errors: as hyena_conv_fwd_ex for the
 * shape and pointers, HYENA_ERR_INVALID_ARG for chunk < 1 or a missing or short workspace,
 * HYENA_ERR_MISALIGNED for a workspace not 256-byte aligned, HYENA_ERR_CUDA when a copy or
 * launch fails (work queued before the failure stays queued).
 */
int hyena_conv_fwd_from_host(const void *q, const void *k, const void *v, const float *h,
                             void *y, int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                             int dtype, int64_t chunk, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/*
 * Host-only: the algorithm (enum hyena_algo, > 0) that HYENA_ALGO_AUTO would run for this
 * problem and these pointers, or minus an error code.  Touches no device.
 */
int hyena_select_algo(const void *q, const void *k, const void *v, const float *h,
                      const void *y, int64_t B, int64_t L, int64_t D, int d_g, int l_h,
                      int l_b, int dtype);

/*
 * Host-only: the bytes of device workspace the backward entry points need for this shape, on
 * any algorithm and any device (a multiple of 256), or minus HYENA_ERR_INVALID_ARG for a bad
 * shape.  The workspace holds fp32 partial filter gradients: on the CUDA-core path one per
 * sequence, 64-step chunk, channel piece and tap; on the register-window path (l_h <= 16) one
 * per thread (a 16-byte channel vector over a run of at least 32 time steps) and tap; on the
 * tensor path one per (CTA, sequence run) and tap, with the run's group and a run count per CTA,
 * and after all partials one 256-byte slot for the tensor path's operand-range flag.
 * Touches no device.  A smaller workspace still runs where it holds what the chosen algorithm
 * needs at least (the window path then takes longer runs); the size returned here runs every
 * algorithm at full speed.
 */
int64_t hyena_conv_bwd_workspace_bytes(int64_t B, int64_t L, int64_t D, int d_g, int l_h);

/*
 * Backward of the gated FIR (the gradients of the two-pass backward of page 04, Sec. 7).  For
 * y = q * z, z = h_g conv x, x = k * v and the upstream gradient dy = dLoss/dy:
 *
 *     dq[b,t,c] = dy[b,t,c] * z[b,t,c]
 *     dx[b,t,c] = sum_{j=0}^{min(l_h-1, L-1-t)} h[c / d_g][j] * q[b,t+j,c] * dy[b,t+j,c]
 *     dk = dx * v,   dv = dx * k
 *     dh[g][j]  = sum_{b, t >= j, c in group g} q[b,t,c] dy[b,t,c] * k[b,t-j,c] v[b,t-j,c]
 *
 * q, k, v, dy, dq, dk, dv: DEVICE [B, L, D] tensors of `dtype`, layout as the forward.
 * h: DEVICE fp32 [D / d_g, l_h].  dh: DEVICE fp32 [D / d_g, l_h], overwritten (not
 * accumulated into).  The forward's shape rules apply (any l_h >= 1).  Algorithm (AUTO): dq
 * comes from the forward kernels (dy in the place of q); where the tensor path applies (bf16,
 * d_g == 64, D % 64 == 0, l_h <= 129, all seven tensors 16-byte aligned) one tcgen05 kernel
 * reads q, k, v, dy once and writes dk, dv once, with fp16 operands (x = k v, dz = q dy, h
 * rounded to fp16) and fp32 accumulation -- where one of them holds a value above 65504, or a
 * group's taps all lie below 2^-10, the kernel raises HYENA_DEVICE_F16_RANGE and fp32
 * CUDA-core kernels queued behind it recompute dk, dv and dh (values of x or dz within fp16's
 * subnormal range, below about 6e-5, take the fp16 path with reduced relative precision);
 * else, for l_h <= 16 with d_g a multiple of 8 (bf16)
 * or 4 (fp32) and q, k, v, dy, dk, dv 16-byte aligned, one CUDA-core register-window kernel
 * (HYENA_ALGO_WINDOW) does the same in fp32; otherwise CUDA-core kernels in fp32 (one for dk,
 * dv, one for the dh partials).  dh is summed in a fixed order on every path: results are
 * deterministic on a given device.
 * workspace: DEVICE scratch of at least hyena_conv_bwd_workspace_bytes() bytes, 16-byte
 * aligned, owned by the caller, unused after the queued work ends.  Outputs must not overlap
 * each other or an input.  B == 0 or L == 0 zeroes dh and launches nothing else.
 * Errors: as the forward, plus HYENA_ERR_INVALID_ARG for a null dy/dk/dv/dh or a workspace
 * that is null or too small, and HYENA_ERR_MISALIGNED for a misaligned dy/dk/dv/dh/workspace.
 */
int hyena_conv_bwd(const void *q, const void *k, const void *v, const float *h, const void *dy,
                   void *dq, void *dk, void *dv, float *dh, int64_t B, int64_t L, int64_t D,
                   int d_g, int l_h, int l_b, int dtype, void *workspace,
                   size_t workspace_bytes, cudaStream_t stream);

/*
 * hyena_conv_bwd with the algorithm chosen by the caller: HYENA_ALGO_AUTO, HYENA_ALGO_TENSOR
 * (the tcgen05 kernel), HYENA_ALGO_WINDOW (the register-window kernel) -- each
 * HYENA_ERR_UNSUPPORTED where it does not apply -- or HYENA_ALGO_DIRECT (the CUDA-core
 * kernels; any shape).  Nothing is queued when an error is returned.
 */
int hyena_conv_bwd_ex(const void *q, const void *k, const void *v, const float *h,
                      const void *dy, void *dq, void *dk, void *dv, float *dh, int64_t B,
                      int64_t L, int64_t D, int d_g, int l_h, int l_b, int dtype, int algo,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Host-only: the algorithm (HYENA_ALGO_TENSOR, HYENA_ALGO_WINDOW or HYENA_ALGO_DIRECT) that
 * HYENA_ALGO_AUTO would run for this backward problem and these pointers, or minus an error
 * code.  Touches no device.
 */
int hyena_select_bwd_algo(const void *q, const void *k, const void *v, const float *h,
                          const void *dy, const void *dq, const void *dk, const void *dv,
                          int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                          int dtype);

/* Size of the fixed device scratch behind hyena_conv_bwd_static_scratch (8 MiB per device). */
#define HYENA_BWD_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * hyena_conv_bwd without a workspace argument.  The pages have no counterpart: this is a
 * convenience of this library.  It is for callers that cannot hand over device memory, such as
 * a C host program with no device allocator of its own, or a runtime that reserves all device
 * memory at start-up and allows no allocation afterwards (cudaMalloc also synchronises the
 * device, which a latency-bound loop cannot afford).  The dh partials go to a fixed array of
 * HYENA_BWD_STATIC_SCRATCH_BYTES in the library's device memory (one per device); this call
 * allocates nothing.  Arguments, results and errors are those of hyena_conv_bwd, plus:
 *   - HYENA_ERR_UNSUPPORTED, with nothing queued, when the least workspace the shape needs
 *     exceeds HYENA_BWD_STATIC_SCRATCH_BYTES (e.g. the D = 4096, d_g = 64, l_h = 128 shape
 *     from B * L = 16384 tokens on: 8 MiB of partials and the range flag); use
 *     hyena_conv_bwd with a workspace there.
 *   - The first call on each device looks up the array's address (cudaGetSymbolAddress) with
 *     that device current and keeps it (a failed lookup returns HYENA_ERR_CUDA and is tried
 *     again on the next call); make that first call before any stream capture.
 *   - Calls that overlap in time on one device (different streams, or threads) share the array
 *     and race: serialise them.  Nothing in the array has to start at zero.
 */
int hyena_conv_bwd_static_scratch(const void *q, const void *k, const void *v, const float *h,
                                  const void *dy, void *dq, void *dk, void *dv, float *dh,
                                  int64_t B, int64_t L, int64_t D, int d_g, int l_h, int l_b,
                                  int dtype, cudaStream_t stream);

/*
 * The l_b x l_b sub-blocks of the lower-triangular Toeplitz matrix of every group
 * (page 04, Sec. 2; index rule of the Sec. 3 worked example):
 *     H_m[g][i][j] = h[g][m*l_b + i - j]  if 0 <= m*l_b + i - j < l_h,  else 0,
 * written for m = 0 (H0), 1 (H1) and 2 (H2) as fp32 [G, l_b, l_b] device arrays.  H2 is the
 * third diagonal that filters with l_h >= l_b + 2 reach; it may be NULL only when
 * l_h <= l_b + 1, where it is all zero.  The forward kernels build their own operand tiles
 * on chip; this entry point exposes the decomposition for inspection and testing.
 * Errors: HYENA_ERR_INVALID_ARG for null h/H0/H1, G < 1, l_h < 1, l_b < 1, l_h > 2*l_b, or
 * H2 == NULL when l_h >= l_b + 2.
 */
int hyena_build_toeplitz(const float *h, float *H0, float *H1, float *H2_or_null, int G,
                         int l_h, int l_b, cudaStream_t stream);

/*
 * Host-only: the number S = 1 + ceil((l_h - 1) / l_b) of sub-block diagonals of the
 * lower-triangular Toeplitz matrix that hold a filter tap (page 04, Sec. 2 block convolution:
 * H_m is zero for m >= S).  Returns minus HYENA_ERR_INVALID_ARG for l_h < 1 or l_b < 1.
 */
int hyena_toeplitz_stages(int l_h, int l_b);

/*
 * All S sub-block diagonals of the block-Toeplitz decomposition (page 04, Sec. 2, with the
 * index rule of the Sec. 3 worked example), for any filter length:
 *     Hm[m][g][i][j] = h[g][m*l_b + i - j]  if 0 <= m*l_b + i - j < l_h,  else 0,
 * for m = 0 .. S-1, written to Hm, a DEVICE fp32 [S, G, l_b, l_b] array owned by the caller.
 * h: DEVICE fp32 [G, l_h].  The decomposition y_n = sum_m H_m x_{n-m} is exact when
 * S >= hyena_toeplitz_stages(l_h, l_b); a smaller S gives the leading diagonals only.
 * Asynchronous on `stream`.  Errors: HYENA_ERR_INVALID_ARG for null h/Hm, S < 1, G < 1,
 * l_h < 1, l_b < 1 or an output too large to index; HYENA_ERR_MISALIGNED for pointers that
 * are not 4-byte aligned; HYENA_ERR_CUDA for a launch failure.
 */
int hyena_build_toeplitz_blocks(const float *h, float *Hm, int S, int G, int l_h, int l_b,
                                cudaStream_t stream);

/*
 * Reads (and, if clear != 0, resets) the status word of the current device: an OR of
 * enum hyena_device_status_bits raised by kernels since the last reset.  Synchronises the
 * current device.  Returns HYENA_OK or HYENA_ERR_CUDA; *out receives the word.
 */
int hyena_device_status(unsigned int *out, int clear);

/* Static description of a status code; never NULL. */
const char *hyena_status_string(int status);

/* ABI version of this header (incremented on incompatible change). */
int hyena_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_CONV_H */
