// complex_scan.cuh -- the selective scan with a complex diagonal A and a
// complex state.
//
// The Mamba-3 page (bitig.info), "Karmaşık Değerli Durum Güncellemesi":
// complex eigenvalues of the state transition let the state rotate and
// oscillate; the page prints no formula.  Reading: A[d][n] = a + i w (a < 0),
// the zero-order hold of "Mamba SSM Nedir? Transformer Alternatifi Rehberi
// (2026)", "Ayrık Zamana Geçiş", in complex arithmetic with real B and C,
// and y from the real part of the state:
//   E    = exp(dt A) - 1                 (Abar = 1 + E)
//   h   <- h + E h + (E / A) B x
//   y    = sum_n C[n] Re h[n] + D x
// E is formed without cancellation for small dt: with s, c = sin, cos of
// dt w / 2 and m = expm1(dt a),
//   Re E = m (1 - 2 s^2) - 2 s^2,   Im E = (1 + m) 2 s c.
// Each step turns the state by dt w: the rotation follows the input through dt.
// When A[n] = (n+1) a + i n w exactly for every state of every channel of a
// warp (the S4D-Lin form), E_{n+1} = E_n + F + E_n F with F = exp(dt (a +
// i w)) - 1 (exp(dt A_{n+1}) = exp(dt A_n) exp(dt (a + i w))): two complex
// exponentials per token and lane instead of one per state, which moves
// the work from the special-function unit to the FMA pipe.
//
// One warp per (batch row, channel group, super-chunk); with 8 or more
// states two lanes share a channel (half of its states each, 16 channels
// per warp, y summed over the pair with one shuffle), which halves the
// registers a lane needs and doubles the warps a shape provides.  Tokens
// are taken in blocks of 32: the warp stages u, dt and the B, C rows
// (converted to fp32) in its shared memory, then steps through the block;
// y goes back through the same buffer.  Sequences are cut into
// super-chunks as in the real scan: an aggregate pass runs each super-chunk
// but the last from a zero state and records its end state and its sum of
// steps (in double: the turn w * sum dt of a long super-chunk must keep its
// fractional part), and the main pass enters super-chunk j with
//   h <- exp(A sum_k) h + h_k      over k < j.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "scan.cuh"

namespace mamba {

constexpr int kCplxWarps = 4;   // jobs per CTA
constexpr int kCplxBlock = 32;  // tokens staged at a time

struct ComplexArgs {
  const void* u;                // (batch, len, channels)
  const void* delta;            // (batch, len, channels)
  const float* A_re;            // (channels, N)
  const float* A_im;            // (channels, N)
  const void* B;                // (batch, len, N)
  const void* C;                // (batch, len, N)
  const float* D;               // (channels) or null
  const float* h0;              // (batch, channels, N, 2) or null
  void* y;                      // (batch, len, channels)
  float* final_state;           // (batch, channels, N, 2) or null
  float* agg_h;                 // (batch, supers-1, channels, N, 2): super-chunk end state from zero
  double* agg_sd;               // (batch, supers-1, channels): its sum of steps
  int64_t len;
  int channels;
  int groups;                   // ceil(channels / channels per warp)
  int supers;
  int64_t super_len;
  int64_t jobs;                 // batch * groups * (supers or supers-1)
};

template <int N>
constexpr int cplx_lanes_per_channel() { return N >= 8 ? 2 : 1; }

template <typename TIO, int N>
struct ComplexSmem {
  static constexpr int kLPC = cplx_lanes_per_channel<N>();
  static constexpr int kCPW = 32 / kLPC;  // channels per warp
  // per warp: u/y and dt [32 tokens][kCPW channels], B and C [32 tokens][N] fp32
  static constexpr int kU = 0;
  static constexpr int kDt = kU + kCplxBlock * kCPW * 4;
  static constexpr int kB = kDt + kCplxBlock * kCPW * 4;
  static constexpr int kC = kB + kCplxBlock * N * 4;
  static constexpr int kWarp = kC + kCplxBlock * N * 4;
  static constexpr int kBytes = kCplxWarps * kWarp;
};

// sin and cos of v after reducing v to [-pi, pi] (|v| < 2^24): the nearest
// integer k to v / (2 pi) by adding and removing 1.5 * 2^23 (on the FMA pipe,
// which leaves the special-function unit to sin and cos)
__device__ __forceinline__ void sincos_reduced(float v, float* s, float* c) {
  const float k = fmaf(v, 0.15915494309189535f, 12582912.0f) - 12582912.0f;
  const float r = fmaf(-k, 6.2831854820251465f, v);          // 2 pi rounded to fp32
  __sincosf(fmaf(k, 1.7484556e-7f, r), s, c);                // + k * (fp32(2 pi) - 2 pi)
}

// exp(x + 2 i v) - 1 without cancellation for small arguments: with s, c =
// sin, cos of v and m = expm1(x),
//   Re = m (1 - 2 s^2) - 2 s^2,   Im = (1 + m) 2 s c.
__device__ __forceinline__ void expm1_complex(float x, float v, float* re, float* im) {
  const float m = expm1_small(x);
  float s, c;
  sincos_reduced(v, &s, &c);
  const float s2 = 2.0f * s * s;
  *re = fmaf(m, 1.0f - s2, -s2);
  *im = (1.0f + m) * (2.0f * s * c);
}

// Stage one B or C row of N values (converted to fp32): 16-byte loads when
// the row allows them, else element by element.
template <typename TIO, int N>
__device__ __forceinline__ void stage_row(float* dst, const TIO* src, bool vec) {
  constexpr int kPer = 16 / (int)sizeof(TIO);  // elements per 16-byte load
  if (vec && (N * (int)sizeof(TIO)) % 16 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += kPer) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + i));
      const TIO* e = reinterpret_cast<const TIO*>(&v);
#pragma unroll
      for (int k = 0; k < kPer; ++k) dst[i + k] = to_f32(e[k]);
    }
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n) dst[n] = to_f32(src[n]);
  }
}

template <typename TIO, int N, bool AGG>
__global__ void __launch_bounds__(kCplxWarps * 32)
complex_scan_kernel(const ComplexArgs a) {
  using L = ComplexSmem<TIO, N>;
  constexpr int LPC = L::kLPC;    // lanes per channel
  constexpr int CPW = L::kCPW;    // channels per warp
  constexpr int NH = N / LPC;     // states per lane
  extern __shared__ __align__(16) unsigned char cplx_smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t job = (int64_t)blockIdx.x * kCplxWarps + warp;
  griddep_wait();  // inputs (and the aggregates) may come from the previous kernel
  if (job >= a.jobs) return;  // whole warp: no block-wide barrier below

  const int per = AGG ? a.supers - 1 : a.supers;
  const int j = (int)(job % per);
  const int64_t bg = job / per;
  const int g = (int)(bg % a.groups);
  const int64_t b = bg / a.groups;
  const int cl = lane / LPC;               // channel of this lane within the warp
  const int n0 = (lane % LPC) * NH;        // first state of this lane
  const int d = CPW * g + cl;
  const bool active = d < a.channels;
  const int dc = active ? d : a.channels - 1;  // inactive lanes read a valid channel, write nothing
  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;

  float* su = reinterpret_cast<float*>(cplx_smem + warp * L::kWarp + L::kU);
  float* sdt = reinterpret_cast<float*>(cplx_smem + warp * L::kWarp + L::kDt);
  float* sB = reinterpret_cast<float*>(cplx_smem + warp * L::kWarp + L::kB);
  float* sC = reinterpret_cast<float*>(cplx_smem + warp * L::kWarp + L::kC);

  // per state: a, w / 2, and 1/A = conj(A) / |A|^2
  float ar[NH], wh[NH], iar[NH], iai[NH];
#pragma unroll
  for (int i = 0; i < NH; ++i) {
    const float re = __ldg(a.A_re + (int64_t)dc * N + n0 + i), im = __ldg(a.A_im + (int64_t)dc * N + n0 + i);
    const float inv = 1.0f / fmaf(re, re, im * im);
    ar[i] = re;
    wh[i] = 0.5f * im;
    iar[i] = re * inv;
    iai[i] = -im * inv;
  }
  // S4D-Lin structure on every channel of the warp: A[n] = (n+1) a + i n w
  // exactly (fp32), i.e. A[n+1] - A[n] = a + i w for all n: then
  // exp(dt A[n+1]) = exp(dt A[n]) exp(dt (a + i w)), and a lane needs two
  // complex exponentials per token instead of one per state
  float sa, sw;  // a and w / 2 of the step a + i w
  bool structured;
  {
    const float a0 = __ldg(a.A_re + (int64_t)dc * N), w1 = N > 1 ? __ldg(a.A_im + (int64_t)dc * N + 1) : 0.0f;
    bool ok = a0 < 0.0f;
    for (int n = 0; n < N; ++n)
      ok &= __ldg(a.A_re + (int64_t)dc * N + n) == (float)(n + 1) * a0 &&
            __ldg(a.A_im + (int64_t)dc * N + n) == (float)n * w1;
    structured = __all_sync(0xffffffffu, ok);
    sa = a0;
    sw = 0.5f * w1;
  }
  float hr[NH], hi[NH];
#pragma unroll
  for (int i = 0; i < NH; ++i) hr[i] = hi[i] = 0.0f;
  if (!AGG) {
    if (a.h0) {
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(a.h0) + ((b * a.channels + dc) * N + n0 + i));
        hr[i] = v.x;
        hi[i] = v.y;
      }
    }
    // enter super-chunk j: h <- exp(A sum_k) h + h_k over the earlier ones
    for (int k = 0; k < j; ++k) {
      const int64_t slot = (b * (a.supers - 1) + k) * a.channels + dc;
      const double sd = a.agg_sd[slot];
      const float2* hk = reinterpret_cast<const float2*>(a.agg_h) + slot * N + n0;
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const float mag = ex2_approx((float)(sd * (double)ar[i]) * 1.4426950408889634f);
        double turn = sd * (2.0 * (double)wh[i]);
        turn -= 6.283185307179586 * rint(turn * 0.15915494309189535);
        float s, c;
        __sincosf((float)turn, &s, &c);
        const float pr = mag * c, pi = mag * s;
        const float2 v = hk[i];
        const float nr = fmaf(pr, hr[i], fmaf(-pi, hi[i], v.x));
        const float ni = fmaf(pr, hi[i], fmaf(pi, hr[i], v.y));
        hr[i] = nr;
        hi[i] = ni;
      }
    }
  }

  const float Dd = (!AGG && a.D) ? __ldg(a.D + dc) : 0.0f;
  // staging: lane = (token row r within a pass of 32/CPW rows, channel c)
  const int sc = lane % CPW, sr = lane / CPW;
  const int dstage = CPW * g + sc < a.channels ? CPW * g + sc : a.channels - 1;
  const TIO* ug = static_cast<const TIO*>(a.u) + b * a.len * a.channels + dstage;
  const TIO* dg = static_cast<const TIO*>(a.delta) + b * a.len * a.channels + dstage;
  const TIO* Bg = static_cast<const TIO*>(a.B) + b * a.len * N;
  const TIO* Cg = static_cast<const TIO*>(a.C) + b * a.len * N;
  TIO* yg = static_cast<TIO*>(a.y) + b * a.len * a.channels + dstage;
  const bool stage_active = CPW * g + sc < a.channels;
  const bool vec = ((reinterpret_cast<uintptr_t>(a.B) | reinterpret_cast<uintptr_t>(a.C)) & 15) == 0;
  double sd_total = 0.0;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kCplxBlock) {
    const int cnt = t_end - t0 < kCplxBlock ? (int)(t_end - t0) : kCplxBlock;
    __syncwarp();
#pragma unroll 4
    for (int k = sr; k < kCplxBlock; k += 32 / CPW) {
      if (k < cnt) {
        su[k * CPW + sc] = to_f32(ug[(t0 + k) * a.channels]);
        sdt[k * CPW + sc] = to_f32(dg[(t0 + k) * a.channels]);
      }
    }
    if (lane < cnt) {
      stage_row<TIO, N>(sB + lane * N, Bg + (t0 + lane) * N, vec);
      if (!AGG) stage_row<TIO, N>(sC + lane * N, Cg + (t0 + lane) * N, vec);
    }
    __syncwarp();
    for (int k = 0; k < cnt; ++k) {
      const float x = su[k * CPW + cl];
      const float dt = sdt[k * CPW + cl];
      sd_total += (double)dt;
      const float* Bt = sB + k * N + n0;
      const float* Ct = sC + k * N + n0;
      float acc = 0.0f;
      // structured: E of the lane's first state and F = exp(dt (a + i w)) - 1
      // from the exponentials, the others by the product chain
      float er = 0.0f, ei = 0.0f, fr = 0.0f, fi = 0.0f;
      if (structured) {
        expm1_complex(dt * ar[0], dt * wh[0], &er, &ei);
        expm1_complex(dt * sa, dt * sw, &fr, &fi);
      }
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        if (!structured) {
          expm1_complex(dt * ar[i], dt * wh[i], &er, &ei);  // exp(dt A) - 1
        } else if (i > 0) {
          // exp(dt A_{n+1}) - 1 = E + F + E F   (exp(dt A_{n+1}) = exp(dt A_n) exp(dt (a + i w)))
          const float nr = er + fr + fmaf(er, fr, -ei * fi);
          const float ni = ei + fi + fmaf(er, fi, ei * fr);
          er = nr;
          ei = ni;
        }
        const float bx = Bt[i] * x;
        const float gr = fmaf(er, iar[i], -ei * iai[i]) * bx;  // Re((E / A) B x)
        const float gi = fmaf(er, iai[i], ei * iar[i]) * bx;   // Im((E / A) B x)
        const float nr = hr[i] + fmaf(er, hr[i], fmaf(-ei, hi[i], gr));
        const float ni = hi[i] + fmaf(er, hi[i], fmaf(ei, hr[i], gi));
        hr[i] = nr;
        hi[i] = ni;
        if (!AGG) acc = fmaf(Ct[i], nr, acc);
      }
      if (!AGG) {
        if (LPC == 2) acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        __syncwarp();  // both lanes of the channel have read x
        if (lane % LPC == 0) su[k * CPW + cl] = fmaf(Dd, x, acc);  // y over x
      }
    }
    if (!AGG) {
      __syncwarp();
      if (stage_active)
        for (int k = sr; k < cnt; k += 32 / CPW) yg[(t0 + k) * a.channels] = from_f32<TIO>(su[k * CPW + sc]);
    }
  }

  griddep_launch_dependents();
  if (!active) return;
  if (AGG) {
    const int64_t slot = (b * (a.supers - 1) + j) * a.channels + d;
    if (lane % LPC == 0) a.agg_sd[slot] = sd_total;
    float2* hk = reinterpret_cast<float2*>(a.agg_h) + slot * N + n0;
#pragma unroll
    for (int i = 0; i < NH; ++i) hk[i] = make_float2(hr[i], hi[i]);
  } else if (a.final_state && j == a.supers - 1) {
    float2* fs = reinterpret_cast<float2*>(a.final_state) + (b * a.channels + d) * N + n0;
#pragma unroll
    for (int i = 0; i < NH; ++i) fs[i] = make_float2(hr[i], hi[i]);
  }
}

}  // namespace mamba
