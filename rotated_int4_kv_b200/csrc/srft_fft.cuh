// srft_fft.cuh -- real DFT of a register-resident vector, for the SRFT of
// "When Quantization Is Free" (gist.science/de/paper/2605.05699, "Methodik" 1-2:
// SRFT(x) = pack(F . diag(s) . x); the FFT passes and the Hermitian unpack into a
// real representation).
//
// The pages run log2(d/2) radix-2 Stockham passes on Metal SIMD groups. Here one
// thread owns a whole vector in registers and runs a radix-2 decimation-in-time
// real FFT whose twiddles are compile-time immediates, so no shuffles and no
// shared-memory passes are needed.
//
// Slot layout of a size-N real spectrum (unnormalised, X_k = sum_n x_n e^{-2 pi i k n/N}):
//   slot 0 = X_0 (DC), slot 1 = X_{N/2} (Nyquist), slot 2k = Re X_k, slot 2k+1 = Im X_k.
// The transform of the samples v[OFF + S*j] (j < N) is written in place: slot j
// lands in v[OFF + S*j]. A size-N stage combines the spectra E (even samples,
// slots at v[OFF + 2S j]) and O (odd samples, at v[OFF + S + 2S j]):
//   X_0 = E_0 + O_0, X_{N/2} = E_0 - O_0, X_{N/4} = E_{N/4} - i O_{N/4},
//   X_k = E_k + W^k O_k, X_{N/2-k} = conj(E_k - W^k O_k), W = e^{-2 pi i / N},
// with the k-butterfly written as four FMAs plus two (a+b, 2a-(a+b)) FMAs.
// rdft_inv is the exact transpose of rdft_fwd (adjoint), so for the orthonormal
// real basis F_r = P Dg A, F_r^T = A^T Dg P^T: decode runs the transpose after
// applying the per-channel normalisation.
#pragma once

#include <cuda_runtime.h>

namespace kvq {

// ---------------------------------------------------------------- compile-time twiddles
// cos / sin of 2 pi m / n, by exact rational octant reduction and a Taylor series
// in double precision (all arguments end up in [0, pi/4]); rounded to float by the caller.
constexpr double kTwoPi = 6.283185307179586476925286766559;

__host__ __device__ constexpr double taylor_sin(double x) {
  double term = x, sum = x;
  const double x2 = x * x;
  for (int i = 1; i < 16; ++i) {
    term *= -x2 / double((2 * i) * (2 * i + 1));
    sum += term;
  }
  return sum;
}

__host__ __device__ constexpr double taylor_cos(double x) {
  double term = 1.0, sum = 1.0;
  const double x2 = x * x;
  for (int i = 1; i < 16; ++i) {
    term *= -x2 / double((2 * i - 1) * (2 * i));
    sum += term;
  }
  return sum;
}

// cos(2 pi m / n) for integers m, n > 0
__host__ __device__ constexpr double cos2pi_frac(long m, long n) {
  m %= n;
  if (m < 0) m += n;
  if (2 * m > n) m = n - m;                      // cos(2pi f) = cos(2pi (1-f)); f in [0, 1/2]
  if (4 * m > n) return -cos2pi_frac(n - 2 * m, 2 * n);  // = -cos(2pi (1/2 - f))
  if (8 * m > n) return taylor_sin(kTwoPi * double(n - 4 * m) / double(4 * n));  // = sin(2pi(1/4 - f))
  return taylor_cos(kTwoPi * double(m) / double(n));
}

__host__ __device__ constexpr double sin2pi_frac(long m, long n) { return cos2pi_frac(n - 4 * m, 4 * n); }

// ---------------------------------------------------------------- butterflies
template <int N, int OFF, int S, int TOT, int K>
struct RdftBfly {
  static __device__ __forceinline__ void fwd(float (&v)[TOT], const float (&e)[N / 2], const float (&o)[N / 2]) {
    if constexpr (K < N / 4) {
      constexpr float c = static_cast<float>(cos2pi_frac(K, N));
      constexpr float s = static_cast<float>(sin2pi_frac(K, N));
      const float er = e[2 * K], ei = e[2 * K + 1], orr = o[2 * K], oi = o[2 * K + 1];
      // W^K O = (c*or + s*oi) + i (c*oi - s*or)
      const float xr = fmaf(c, orr, fmaf(s, oi, er));
      const float xi = fmaf(c, oi, fmaf(-s, orr, ei));
      v[OFF + S * (2 * K)] = xr;
      v[OFF + S * (2 * K + 1)] = xi;
      v[OFF + S * (N - 2 * K)] = fmaf(2.0f, er, -xr);      // Re(E - W O)
      v[OFF + S * (N - 2 * K + 1)] = fmaf(-2.0f, ei, xi);  // -Im(E - W O)
      RdftBfly<N, OFF, S, TOT, K + 1>::fwd(v, e, o);
    }
  }
  static __device__ __forceinline__ void inv(const float (&v)[TOT], float (&e)[N / 2], float (&o)[N / 2]) {
    if constexpr (K < N / 4) {
      constexpr float c = static_cast<float>(cos2pi_frac(K, N));
      constexpr float s = static_cast<float>(sin2pi_frac(K, N));
      const float ar = v[OFF + S * (2 * K)], ai = v[OFF + S * (2 * K + 1)];
      const float br = v[OFF + S * (N - 2 * K)], bi = v[OFF + S * (N - 2 * K + 1)];
      e[2 * K] = ar + br;
      e[2 * K + 1] = ai - bi;
      const float dr = ar - br, di = ai + bi;
      o[2 * K] = fmaf(c, dr, -s * di);
      o[2 * K + 1] = fmaf(s, dr, c * di);
      RdftBfly<N, OFF, S, TOT, K + 1>::inv(v, e, o);
    }
  }
};

template <int N, int OFF, int S, int TOT>
struct Rdft {
  static_assert(N >= 4 && (N & (N - 1)) == 0, "N must be a power of two >= 4");
  static __device__ __forceinline__ void fwd(float (&v)[TOT]) {
    Rdft<N / 2, OFF, 2 * S, TOT>::fwd(v);
    Rdft<N / 2, OFF + S, 2 * S, TOT>::fwd(v);
    constexpr int M = N / 2;
    float e[M], o[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      e[j] = v[OFF + 2 * S * j];
      o[j] = v[OFF + S + 2 * S * j];
    }
    v[OFF] = e[0] + o[0];
    v[OFF + S] = e[0] - o[0];
    v[OFF + S * M] = e[1];
    v[OFF + S * (M + 1)] = -o[1];
    RdftBfly<N, OFF, S, TOT, 1>::fwd(v, e, o);
  }
  static __device__ __forceinline__ void inv(float (&v)[TOT]) {
    constexpr int M = N / 2;
    float e[M], o[M];
    const float x0 = v[OFF], xn = v[OFF + S];
    e[0] = x0 + xn;
    o[0] = x0 - xn;
    e[1] = v[OFF + S * M];
    o[1] = -v[OFF + S * (M + 1)];
    RdftBfly<N, OFF, S, TOT, 1>::inv(v, e, o);
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[OFF + 2 * S * j] = e[j];
      v[OFF + S + 2 * S * j] = o[j];
    }
    Rdft<N / 2, OFF, 2 * S, TOT>::inv(v);
    Rdft<N / 2, OFF + S, 2 * S, TOT>::inv(v);
  }
};

template <int OFF, int S, int TOT>
struct Rdft<2, OFF, S, TOT> {
  static __device__ __forceinline__ void fwd(float (&v)[TOT]) {
    const float a = v[OFF], b = v[OFF + S];
    v[OFF] = a + b;
    v[OFF + S] = a - b;
  }
  static __device__ __forceinline__ void inv(float (&v)[TOT]) { fwd(v); }
};

// Whole-vector transforms: slots of the size-N spectrum in v[0..N).
template <int N>
__device__ __forceinline__ void rdft_fwd(float (&v)[N]) {
  Rdft<N, 0, 1, N>::fwd(v);
}
template <int N>
__device__ __forceinline__ void rdft_inv(float (&v)[N]) {
  Rdft<N, 0, 1, N>::inv(v);
}

// ---------------------------------------------------------------- packed (f32x2) transforms
// Two independent real sequences per float2 (.x and .y); every butterfly runs as
// Blackwell packed fp32 instructions (fma/add/sub .f32x2), i.e. one issue slot
// for two scalar operations. Used for the two halves of the first decimation:
// with v[m] = (x[2m], x[2m+1]), a packed size-N/2 transform gives E (even
// samples) in .x and O (odd samples) in .y; rdft_top_* then forms the size-N
// spectrum with scalar butterflies.
__device__ __forceinline__ float2 p2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 p2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 p2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 p2sub(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 p2bc(float x) { return make_float2(x, x); }

template <int N, int OFF, int S, int TOT, int K>
struct RdftBflyP {
  static __device__ __forceinline__ void fwd(float2 (&v)[TOT], const float2 (&e)[N / 2], const float2 (&o)[N / 2]) {
    if constexpr (K < N / 4) {
      constexpr float c = static_cast<float>(cos2pi_frac(K, N));
      constexpr float s = static_cast<float>(sin2pi_frac(K, N));
      const float2 er = e[2 * K], ei = e[2 * K + 1], orr = o[2 * K], oi = o[2 * K + 1];
      const float2 xr = p2fma(p2bc(c), orr, p2fma(p2bc(s), oi, er));
      const float2 xi = p2fma(p2bc(c), oi, p2fma(p2bc(-s), orr, ei));
      v[OFF + S * (2 * K)] = xr;
      v[OFF + S * (2 * K + 1)] = xi;
      v[OFF + S * (N - 2 * K)] = p2fma(p2bc(-c), orr, p2fma(p2bc(-s), oi, er));  // Re(E - W O)
      v[OFF + S * (N - 2 * K + 1)] = p2fma(p2bc(-2.0f), ei, xi);                 // -Im(E - W O)
      RdftBflyP<N, OFF, S, TOT, K + 1>::fwd(v, e, o);
    }
  }
  static __device__ __forceinline__ void inv(const float2 (&v)[TOT], float2 (&e)[N / 2], float2 (&o)[N / 2]) {
    if constexpr (K < N / 4) {
      constexpr float c = static_cast<float>(cos2pi_frac(K, N));
      constexpr float s = static_cast<float>(sin2pi_frac(K, N));
      const float2 ar = v[OFF + S * (2 * K)], ai = v[OFF + S * (2 * K + 1)];
      const float2 br = v[OFF + S * (N - 2 * K)], bi = v[OFF + S * (N - 2 * K + 1)];
      e[2 * K] = p2add(ar, br);
      e[2 * K + 1] = p2sub(ai, bi);
      const float2 dr = p2sub(ar, br), di = p2add(ai, bi);
      o[2 * K] = p2fma(p2bc(c), dr, p2mul(p2bc(-s), di));
      o[2 * K + 1] = p2fma(p2bc(s), dr, p2mul(p2bc(c), di));
      RdftBflyP<N, OFF, S, TOT, K + 1>::inv(v, e, o);
    }
  }
};

template <int N, int OFF, int S, int TOT>
struct RdftP {
  static_assert(N >= 4 && (N & (N - 1)) == 0, "N must be a power of two >= 4");
  static __device__ __forceinline__ void fwd(float2 (&v)[TOT]) {
    RdftP<N / 2, OFF, 2 * S, TOT>::fwd(v);
    RdftP<N / 2, OFF + S, 2 * S, TOT>::fwd(v);
    constexpr int M = N / 2;
    float2 e[M], o[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      e[j] = v[OFF + 2 * S * j];
      o[j] = v[OFF + S + 2 * S * j];
    }
    v[OFF] = p2add(e[0], o[0]);
    v[OFF + S] = p2sub(e[0], o[0]);
    v[OFF + S * M] = e[1];
    v[OFF + S * (M + 1)] = p2sub(make_float2(0.0f, 0.0f), o[1]);
    RdftBflyP<N, OFF, S, TOT, 1>::fwd(v, e, o);
  }
  static __device__ __forceinline__ void inv(float2 (&v)[TOT]) {
    constexpr int M = N / 2;
    float2 e[M], o[M];
    const float2 x0 = v[OFF], xn = v[OFF + S];
    e[0] = p2add(x0, xn);
    o[0] = p2sub(x0, xn);
    e[1] = v[OFF + S * M];
    o[1] = p2sub(make_float2(0.0f, 0.0f), v[OFF + S * (M + 1)]);
    RdftBflyP<N, OFF, S, TOT, 1>::inv(v, e, o);
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[OFF + 2 * S * j] = e[j];
      v[OFF + S + 2 * S * j] = o[j];
    }
    RdftP<N / 2, OFF, 2 * S, TOT>::inv(v);
    RdftP<N / 2, OFF + S, 2 * S, TOT>::inv(v);
  }
};

template <int OFF, int S, int TOT>
struct RdftP<2, OFF, S, TOT> {
  static __device__ __forceinline__ void fwd(float2 (&v)[TOT]) {
    const float2 a = v[OFF], b = v[OFF + S];
    v[OFF] = p2add(a, b);
    v[OFF + S] = p2sub(a, b);
  }
  static __device__ __forceinline__ void inv(float2 (&v)[TOT]) { fwd(v); }
};

// Top stage (scalar) of a size-N transform whose even/odd halves were transformed
// packed: in v[j] = (E slot j, O slot j), out v[k] = (Re X_k, Im X_k) for
// 1 <= k < N/2 and v[0] = (X_0, X_{N/2}) -- the same slot order as rdft_fwd.
template <int N, int K>
__device__ __forceinline__ void rdft_top_bfly(float2 (&v)[N / 2], const float (&e)[N / 2], const float (&o)[N / 2]) {
  if constexpr (K < N / 4) {
    constexpr float c = static_cast<float>(cos2pi_frac(K, N));
    constexpr float s = static_cast<float>(sin2pi_frac(K, N));
    const float er = e[2 * K], ei = e[2 * K + 1], orr = o[2 * K], oi = o[2 * K + 1];
    const float xr = fmaf(c, orr, fmaf(s, oi, er));
    const float xi = fmaf(c, oi, fmaf(-s, orr, ei));
    v[K] = make_float2(xr, xi);
    v[N / 2 - K] = make_float2(fmaf(2.0f, er, -xr), fmaf(-2.0f, ei, xi));
    rdft_top_bfly<N, K + 1>(v, e, o);
  }
}

template <int N>
__device__ __forceinline__ void rdft_fwd_packed(float2 (&v)[N / 2]) {
  RdftP<N / 2, 0, 1, N / 2>::fwd(v);
  float e[N / 2], o[N / 2];
#pragma unroll
  for (int j = 0; j < N / 2; ++j) {
    e[j] = v[j].x;
    o[j] = v[j].y;
  }
  v[0] = make_float2(e[0] + o[0], e[0] - o[0]);
  v[N / 4] = make_float2(e[1], -o[1]);
  rdft_top_bfly<N, 1>(v, e, o);
}

// Exact transpose of rdft_fwd_packed: slots in, (x[2m], x[2m+1]) pairs out.
template <int N, int K>
__device__ __forceinline__ void rdft_top_bfly_inv(const float2 (&v)[N / 2], float (&e)[N / 2], float (&o)[N / 2]) {
  if constexpr (K < N / 4) {
    constexpr float c = static_cast<float>(cos2pi_frac(K, N));
    constexpr float s = static_cast<float>(sin2pi_frac(K, N));
    const float ar = v[K].x, ai = v[K].y, br = v[N / 2 - K].x, bi = v[N / 2 - K].y;
    e[2 * K] = ar + br;
    e[2 * K + 1] = ai - bi;
    const float dr = ar - br, di = ai + bi;
    o[2 * K] = fmaf(c, dr, -s * di);
    o[2 * K + 1] = fmaf(s, dr, c * di);
    rdft_top_bfly_inv<N, K + 1>(v, e, o);
  }
}

template <int N>
__device__ __forceinline__ void rdft_inv_packed(float2 (&v)[N / 2]) {
  float e[N / 2], o[N / 2];
  e[0] = v[0].x + v[0].y;
  o[0] = v[0].x - v[0].y;
  e[1] = v[N / 4].x;
  o[1] = -v[N / 4].y;
  rdft_top_bfly_inv<N, 1>(v, e, o);
#pragma unroll
  for (int j = 0; j < N / 2; ++j) v[j] = make_float2(e[j], o[j]);
  RdftP<N / 2, 0, 1, N / 2>::inv(v);
}

// D = 256 pair combine: thread p of a pair holds the size-128 spectrum of the samples
// x[2j + p] (E for p = 0, O for p = 1) in slot order; it forms X_k and X_{128-k} for
// k = 32p + J, J = 0..32, exchanging one value per component with its partner.
// Thread 0 then owns channels [0, 64) and [192, 256), thread 1 channels [64, 192);
// local value L of both threads maps to the same (J, X or X_{128-k}, Re or Im), except L = 0.
template <int S_>
struct TwPair {  // W_256^(32p + J) for p = 0, 1
  static constexpr float c0 = static_cast<float>(cos2pi_frac(S_, 256));
  static constexpr float s0 = static_cast<float>(sin2pi_frac(S_, 256));
  static constexpr float c1 = static_cast<float>(cos2pi_frac(S_ + 32, 256));
  static constexpr float s1 = static_cast<float>(sin2pi_frac(S_ + 32, 256));
};

__device__ __forceinline__ float slotv(const float2 (&u)[64], int sl) { return (sl & 1) ? u[sl >> 1].y : u[sl >> 1].x; }
__device__ __forceinline__ void slot_add(float2 (&u)[64], int sl, float v) {
  if (sl & 1)
    u[sl >> 1].y += v;
  else
    u[sl >> 1].x += v;
}

template <int J>
__device__ __forceinline__ void pair_combine(const float2 (&u)[64], float (&o)[128], const bool p) {
  if constexpr (J <= 32) {
    constexpr int k0 = J, k1 = 32 + J;
    constexpr int re0 = k0 == 0 ? 0 : 2 * k0, im0 = k0 == 0 ? -1 : 2 * k0 + 1;
    constexpr int re1 = k1 == 64 ? 1 : 2 * k1, im1 = k1 == 64 ? -1 : 2 * k1 + 1;
    const float u_re0 = slotv(u, re0), u_re1 = slotv(u, re1);
    const float u_im0 = im0 < 0 ? 0.0f : slotv(u, im0 < 0 ? 0 : im0);
    const float u_im1 = im1 < 0 ? 0.0f : slotv(u, im1 < 0 ? 0 : im1);
    const float mine_re = p ? u_re1 : u_re0, send_re = p ? u_re0 : u_re1;
    const float mine_im = p ? u_im1 : u_im0, send_im = p ? u_im0 : u_im1;
    const float recv_re = __shfl_xor_sync(0xffffffffu, send_re, 1);
    const float recv_im = __shfl_xor_sync(0xffffffffu, send_im, 1);
    const float er = p ? recv_re : mine_re, ei = p ? recv_im : mine_im;
    const float orr = p ? mine_re : recv_re, oi = p ? mine_im : recv_im;
    const float c = p ? TwPair<J>::c1 : TwPair<J>::c0;
    const float sn = p ? TwPair<J>::s1 : TwPair<J>::s0;
    const float xr = fmaf(c, orr, fmaf(sn, oi, er));  // X_k = E + W O
    const float xi = fmaf(c, oi, fmaf(-sn, orr, ei));
    const float yr = fmaf(2.0f, er, -xr);              // X_{128-k} = conj(E - W O)
    const float yi = fmaf(-2.0f, ei, xi);
    if constexpr (J == 0) {
      o[0] = p ? xi : xr;
      o[127] = yr;
    } else if constexpr (J < 32) {
      o[2 * J - 1] = xr;
      o[2 * J] = xi;
      o[127 - 2 * J] = yr;
      o[128 - 2 * J] = yi;
    } else {
      o[63] = xr;
      o[64] = yi;
    }
    pair_combine<J + 1>(u, o, p);
  }
}


// Exact transpose of pair_combine: local values in (same placement), slots of the
// thread's size-128 spectrum out (u must be zeroed by the caller; the slots of
// k = 32 receive one contribution from each of J = 0 and J = 32).
template <int J>
__device__ __forceinline__ void pair_combine_inv(const float (&o)[128], float2 (&u)[64], const bool p) {
  if constexpr (J <= 32) {
    constexpr int k0 = J, k1 = 32 + J;
    constexpr int re0 = k0 == 0 ? 0 : 2 * k0, im0 = k0 == 0 ? -1 : 2 * k0 + 1;
    constexpr int re1 = k1 == 64 ? 1 : 2 * k1, im1 = k1 == 64 ? -1 : 2 * k1 + 1;
    float xr, xi, yr, yi;
    if constexpr (J == 0) {
      xr = p ? 0.0f : o[0];
      xi = p ? o[0] : 0.0f;
      yr = o[127];
      yi = 0.0f;
    } else if constexpr (J < 32) {
      xr = o[2 * J - 1];
      xi = o[2 * J];
      yr = o[127 - 2 * J];
      yi = o[128 - 2 * J];
    } else {
      xr = o[63];
      xi = 0.0f;
      yr = 0.0f;
      yi = o[64];
    }
    const float c = p ? TwPair<J>::c1 : TwPair<J>::c0;
    const float sn = p ? TwPair<J>::s1 : TwPair<J>::s0;
    const float er = xr + yr, ei = xi - yi;
    const float dr = xr - yr, di = xi + yi;
    const float orr = fmaf(c, dr, -sn * di), oi = fmaf(sn, dr, c * di);
    const float mine_re = p ? orr : er, mine_im = p ? oi : ei;
    const float rb_re = p ? er : orr, rb_im = p ? ei : oi;
    const float send_re = __shfl_xor_sync(0xffffffffu, rb_re, 1);
    const float send_im = __shfl_xor_sync(0xffffffffu, rb_im, 1);
    const float a_re1 = p ? mine_re : send_re, a_re0 = p ? send_re : mine_re;
    const float a_im1 = p ? mine_im : send_im, a_im0 = p ? send_im : mine_im;
    slot_add(u, re0, a_re0);
    slot_add(u, re1, a_re1);
    if constexpr (im0 >= 0) slot_add(u, im0, a_im0);
    if constexpr (im1 >= 0) slot_add(u, im1, a_im1);
    pair_combine_inv<J + 1>(o, u, p);
  }
}

// Rotated channel c (DC, cos1, sin1, ..., Nyquist order) <-> spectrum slot.
__host__ __device__ constexpr int slot_of_channel(int c, int N) { return c == 0 ? 0 : (c == N - 1 ? 1 : c + 1); }

}  // namespace kvq
