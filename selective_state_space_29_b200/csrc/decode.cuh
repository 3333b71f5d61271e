// decode.cuh -- the single-token recurrent state update (generation mode).
//
// Page "Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)": the
// recurrence of section "Ayrık Zamana Geçiş" applied to one new token, on the
// fixed-size state that section "Karmaşıklık Karşılaştırması" contrasts with
// a transformer's growing cache.  Per (batch b, channel d) row and state n:
//     e      = exp(Delta A_n) - 1
//     h_n   <- (1 + e) h_n + (e / A_n) B_n x        (= Abar h + Bbar x)
//     y      = sum_n C_n h_n + D x
//
// The kernel is bound by HBM traffic: each update reads and writes the row's
// N fp32 states (128 bytes at N = 16) and touches only a few bytes more.
// Layout: NS/4 consecutive lanes share one row, each holding four states as
// one float4, so a warp moves 512 contiguous bytes per access.  A thread
// keeps its channel's A and D in registers and walks ROWS batch rows, whose
// loads are all issued before any arithmetic (ROWS x 16 bytes of state in
// flight per thread).
#pragma once

#include "common.cuh"
#include "scan.cuh"  // expm1_small / expm1_fast

namespace mamba {

template <typename TIO, int NS>
struct DecodeArgs {
  float* __restrict__ state;
  const TIO* __restrict__ x;
  const TIO* __restrict__ delta;
  const float* __restrict__ A;
  const TIO* __restrict__ B;
  const TIO* __restrict__ C;
  const float* __restrict__ D;
  TIO* __restrict__ y;
  int64_t batch, channels;
};

template <typename TIO>
__device__ __forceinline__ void load4(const TIO* p, float (&v)[4]) {
  if constexpr (sizeof(TIO) == 4) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xffff0000u);
  }
}

constexpr int kDecodeWarps = 8;  // warps per CTA

// grid: x over channel tiles of kDecodeWarps * 32 / (NS/4) channels,
//       y over batch tiles of ROWS batch rows.
// FASTQ: exp(z) - 1 from the hardware exp2 (bf16 data); otherwise the
// branch-free accurate form.
template <typename TIO, int NS, int ROWS, bool FASTQ>
__global__ void __launch_bounds__(kDecodeWarps * 32, 1)
state_update_kernel(const DecodeArgs<TIO, NS> a) {
  constexpr int QPR = NS / 4;           // lanes per row
  constexpr int CPW = 32 / QPR;         // channels per warp
  static_assert(32 % QPR == 0, "a row must not straddle a warp");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int q = lane % QPR;
  const int64_t d = ((int64_t)blockIdx.x * kDecodeWarps + warp) * CPW + lane / QPR;
  const bool dok = d < a.channels;
  const int64_t b0 = (int64_t)blockIdx.y * ROWS;
  // the next step's kernel may be scheduled as this one's CTAs retire; every
  // input of this one may come from the previous kernel of the stream
  griddep_launch_dependents();
  griddep_wait();

  float av[4] = {-1.f, -1.f, -1.f, -1.f};
  float Dd = 0.0f;
  if (dok) {
    const float4 A4 = __ldg(reinterpret_cast<const float4*>(a.A + d * NS) + q);
    av[0] = A4.x; av[1] = A4.y; av[2] = A4.z; av[3] = A4.w;
    Dd = a.D ? __ldg(a.D + d) : 0.0f;
  }
  float inva[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) inva[i] = 1.0f / av[i];
  // A[d][n] = (n+1) A[d][0] on every channel of the warp: a lane's four
  // exp(Delta A_n) - 1 follow from two exponentials, that of its first state
  // and that of A[d][0], by e_{n+1} = e^{Delta A_0} e_n + (e^{Delta A_0} - 1)
  float a0 = -1.0f;
  bool st_ok = true;
  if (dok) {
    a0 = __ldg(a.A + d * NS);
#pragma unroll
    for (int i = 0; i < 4; ++i) st_ok &= av[i] == (float)(4 * q + i + 1) * a0;
    st_ok &= a0 < 0.0f;
  }
  const bool structured = __all_sync(0xffffffffu, st_ok);
  const float a_first = (float)(4 * q + 1) * a0;

  // issue every load first
  float4 h[ROWS];
  float bv[ROWS][4], cv[ROWS][4], xv[ROWS], dv[ROWS];
  bool ok[ROWS];
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    const int64_t b = b0 + k;
    ok[k] = dok && b < a.batch;
    const int64_t r = ok[k] ? b * a.channels + d : 0;
    const int64_t bb = ok[k] ? b : 0;
    h[k] = ok[k] ? reinterpret_cast<const float4*>(a.state + r * NS)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    load4<TIO>(a.B + bb * NS + 4 * q, bv[k]);
    load4<TIO>(a.C + bb * NS + 4 * q, cv[k]);
    xv[k] = ok[k] ? to_f32(a.x[r]) : 0.0f;
    dv[k] = ok[k] ? to_f32(a.delta[r]) : 0.0f;
  }
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    float hv[4] = {h[k].x, h[k].y, h[k].z, h[k].w};
    float acc = 0.0f;
    float ev[4];
    if (structured) {
      const float z0 = dv[k] * a0;
      const float q0 = FASTQ ? expm1_fast(z0) : expm1_small(z0);
      const float r0 = 1.0f + q0;
      ev[0] = FASTQ ? expm1_fast(dv[k] * a_first) : expm1_small(dv[k] * a_first);
#pragma unroll
      for (int i = 1; i < 4; ++i) ev[i] = fmaf(r0, ev[i - 1], q0);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float z = dv[k] * av[i];
        ev[i] = FASTQ ? expm1_fast(z) : expm1_small(z);   // exp(Delta A_n) - 1
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float e = ev[i];
      const float phi = e * inva[i];              // (Delta A_n)^-1 (exp(Delta A_n) - 1) Delta
      hv[i] = fmaf(phi, bv[k][i] * xv[k], fmaf(e, hv[i], hv[i]));
      acc = fmaf(cv[k][i], hv[i], acc);
    }
#pragma unroll
    for (int off = 1; off < QPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (ok[k]) {
      const int64_t r = (b0 + k) * a.channels + d;
      reinterpret_cast<float4*>(a.state + r * NS)[q] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      if (q == 0) a.y[r] = from_f32<TIO>(fmaf(Dd, xv[k], acc));
    }
  }
}

// ---------------------------------------------------------------------------
// Multi-input multi-output state update (the Mamba-3 page, "MIMO
// Mekanizmasının İşleyişi": one state update per step serves several
// outputs).  Per (batch b, channel d) row, R inputs x^(r) and R outputs:
//     h_n   <- (1 + e) h_n + (e / A_n) sum_r B^(r)_n x^(r)
//     y^(r)  = sum_n C^(r)_n h_n + D x^(r)
// x, y [batch][R][channels]; B, C [batch][R][NS].  The state is read and
// written once for R outputs, so the bytes per output fall by about R.
// Same lane layout as state_update_kernel (NS/4 lanes per row, a float4
// of states each); lane q of a row writes output q (R <= NS/4).
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int R, int ROWS, bool FASTQ>
__global__ void __launch_bounds__(kDecodeWarps * 32, 1)
state_update_mimo_kernel(const DecodeArgs<TIO, NS> a) {
  constexpr int QPR = NS / 4;
  constexpr int CPW = 32 / QPR;
  static_assert(32 % QPR == 0 && R <= QPR, "a row's outputs are written by its own lanes");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int q = lane % QPR;
  const int64_t d = ((int64_t)blockIdx.x * kDecodeWarps + warp) * CPW + lane / QPR;
  const bool dok = d < a.channels;
  const int64_t b0 = (int64_t)blockIdx.y * ROWS;
  griddep_launch_dependents();
  griddep_wait();

  float av[4] = {-1.f, -1.f, -1.f, -1.f};
  float Dd = 0.0f;
  if (dok) {
    const float4 A4 = __ldg(reinterpret_cast<const float4*>(a.A + d * NS) + q);
    av[0] = A4.x; av[1] = A4.y; av[2] = A4.z; av[3] = A4.w;
    Dd = a.D ? __ldg(a.D + d) : 0.0f;
  }
  float inva[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) inva[i] = 1.0f / av[i];
  // structured A on every channel of the warp: two exponentials per lane and
  // the chain e_{n+1} = e^{Delta A_0} e_n + (e^{Delta A_0} - 1), as in state_update_kernel
  float a0 = -1.0f;
  bool st_ok = true;
  if (dok) {
    a0 = __ldg(a.A + d * NS);
#pragma unroll
    for (int i = 0; i < 4; ++i) st_ok &= av[i] == (float)(4 * q + i + 1) * a0;
    st_ok &= a0 < 0.0f;
  }
  const bool structured = __all_sync(0xffffffffu, st_ok);
  const float a_first = (float)(4 * q + 1) * a0;

  float4 h[ROWS];
  float bv[ROWS][R][4], cv[ROWS][R][4], xv[ROWS][R], dv[ROWS];
  bool ok[ROWS];
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    const int64_t b = b0 + k;
    ok[k] = dok && b < a.batch;
    const int64_t bb = ok[k] ? b : 0;
    const int64_t r = ok[k] ? b * a.channels + d : 0;
    h[k] = ok[k] ? reinterpret_cast<const float4*>(a.state + r * NS)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    dv[k] = ok[k] ? to_f32(a.delta[r]) : 0.0f;
#pragma unroll
    for (int j = 0; j < R; ++j) {
      load4<TIO>(a.B + (bb * R + j) * NS + 4 * q, bv[k][j]);
      load4<TIO>(a.C + (bb * R + j) * NS + 4 * q, cv[k][j]);
      xv[k][j] = ok[k] ? to_f32(a.x[(bb * R + j) * a.channels + d]) : 0.0f;
    }
  }
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    float hv[4] = {h[k].x, h[k].y, h[k].z, h[k].w};
    float acc[R];
#pragma unroll
    for (int j = 0; j < R; ++j) acc[j] = 0.0f;
    float ev[4];
    if (structured) {
      const float z0 = dv[k] * a0;
      const float q0 = FASTQ ? expm1_fast(z0) : expm1_small(z0);
      const float r0 = 1.0f + q0;
      ev[0] = FASTQ ? expm1_fast(dv[k] * a_first) : expm1_small(dv[k] * a_first);
#pragma unroll
      for (int i = 1; i < 4; ++i) ev[i] = fmaf(r0, ev[i - 1], q0);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) ev[i] = FASTQ ? expm1_fast(dv[k] * av[i]) : expm1_small(dv[k] * av[i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float e = ev[i];
      float in = 0.0f;
#pragma unroll
      for (int j = 0; j < R; ++j) in = fmaf(bv[k][j][i], xv[k][j], in);
      hv[i] = fmaf(e * inva[i], in, fmaf(e, hv[i], hv[i]));
#pragma unroll
      for (int j = 0; j < R; ++j) acc[j] = fmaf(cv[k][j][i], hv[i], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < R; ++j)
#pragma unroll
      for (int off = 1; off < QPR; off <<= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    if (ok[k]) {
      const int64_t b = b0 + k;
      reinterpret_cast<float4*>(a.state + (b * a.channels + d) * NS)[q] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      float mine = 0.0f, xm = 0.0f;
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (q == j) {
          mine = acc[j];
          xm = xv[k][j];
        }
      if (q < R) a.y[(b * R + q) * a.channels + d] = from_f32<TIO>(fmaf(Dd, xm, mine));
    }
  }
}

}  // namespace mamba
