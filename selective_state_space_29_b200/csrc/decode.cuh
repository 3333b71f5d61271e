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
// one float4, so a warp moves 512 contiguous bytes per access.
#pragma once

#include "common.cuh"

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
    v[0] = p[0]; v[1] = p[1]; v[2] = p[2]; v[3] = p[3];
  } else {
    const __nv_bfloat162 lo = reinterpret_cast<const __nv_bfloat162*>(p)[0];
    const __nv_bfloat162 hi = reinterpret_cast<const __nv_bfloat162*>(p)[1];
    v[0] = __low2float(lo); v[1] = __high2float(lo);
    v[2] = __low2float(hi); v[3] = __high2float(hi);
  }
}

template <typename TIO, int NS, int ROWS_PER_THREAD>
__global__ void __launch_bounds__(256)
state_update_kernel(const DecodeArgs<TIO, NS> a) {
  constexpr int QPR = NS / 4;  // lanes per row
  static_assert(32 % QPR == 0, "a row must not straddle a warp");
  constexpr int RPW = 32 / QPR;  // rows per warp access
  const int64_t rows = a.batch * a.channels;
  const int lane = threadIdx.x & 31;
  const int q = lane % QPR;
  const int lane_row = lane / QPR;
  const int64_t warp_g = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;

  // the loop bound is uniform across the warp (the shuffles below need it)
  for (int64_t wb = warp_g; wb * RPW < rows; wb += nwarps * ROWS_PER_THREAD) {
    float4 h[ROWS_PER_THREAD];
    float av[ROWS_PER_THREAD][4], bv[ROWS_PER_THREAD][4], cv[ROWS_PER_THREAD][4];
    float xv[ROWS_PER_THREAD], dv[ROWS_PER_THREAD], Dd[ROWS_PER_THREAD];
    bool ok[ROWS_PER_THREAD];
    // issue every load first (two rows in flight per thread)
#pragma unroll
    for (int k = 0; k < ROWS_PER_THREAD; ++k) {
      const int64_t r = (wb + (int64_t)k * nwarps) * RPW + lane_row;
      ok[k] = r < rows;
      const int64_t rr = ok[k] ? r : 0;
      const int64_t b = rr / a.channels;
      const int64_t d = rr - b * a.channels;
      h[k] = reinterpret_cast<const float4*>(a.state + rr * NS)[q];
      const float4 A4 = __ldg(reinterpret_cast<const float4*>(a.A + d * NS) + q);
      av[k][0] = A4.x; av[k][1] = A4.y; av[k][2] = A4.z; av[k][3] = A4.w;
      load4<TIO>(a.B + b * NS + 4 * q, bv[k]);
      load4<TIO>(a.C + b * NS + 4 * q, cv[k]);
      xv[k] = to_f32(a.x[rr]);
      dv[k] = to_f32(a.delta[rr]);
      Dd[k] = a.D ? __ldg(a.D + d) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < ROWS_PER_THREAD; ++k) {
      float hv[4] = {h[k].x, h[k].y, h[k].z, h[k].w};
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float z = dv[k] * av[k][i];
        const float e = expm1_neg(z);                     // exp(Delta A_n) - 1
        const float phi = (av[k][i] != 0.0f) ? e / av[k][i] : dv[k];  // (Delta A)^-1 (e^{Delta A} - 1) Delta
        hv[i] = fmaf(phi, bv[k][i] * xv[k], fmaf(e, hv[i], hv[i]));
        acc = fmaf(cv[k][i], hv[i], acc);
      }
#pragma unroll
      for (int off = 1; off < QPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (ok[k]) {
        const int64_t r = (wb + (int64_t)k * nwarps) * RPW + lane_row;
        reinterpret_cast<float4*>(a.state + r * NS)[q] = make_float4(hv[0], hv[1], hv[2], hv[3]);
        if (q == 0) a.y[r] = from_f32<TIO>(fmaf(Dd[k], xv[k], acc));
      }
    }
  }
}

}  // namespace mamba
