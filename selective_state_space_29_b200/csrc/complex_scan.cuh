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
// warp (the S4D-Lin form), exp(dt A_{n+1}) = exp(dt A_n) exp(dt (a + i w)):
// with F = exp(dt (a + i w)) - 1 and F2 = exp(2 dt (a + i w)) - 1 = F (2 + F),
// E_0 = expm1(dt a) (A_0 is real), E_1 = E_0 + F + E_0 F and
// E_{n+2} = E_n + F2 + E_n F2, which walks two states at a time: two
// exponentials per token and lane instead of one per state.  That path keeps
// the state scaled, g = A h, as the real scan does:
//   g <- g + E (g + B x),      Re h = Re(g / A),
// and holds pairs of states in float2 registers so that the chain, the
// update and the output are packed FFMA2 (about 7.5 per state).
//
// One warp per (batch row, channel group, super-chunk); with 8 or more
// states two lanes share a channel (half of its states each, 16 channels per
// warp, y summed over the pair with one shuffle), which doubles the warps a
// shape provides.  Tokens are taken in blocks of 32: while the warp steps
// through one block, the next one's u, dt, B and C rows are in flight to its
// shared memory (16-byte cp.async copies into the other half of a double
// buffer; plain loads when rows are not 16-byte pieces).  B and C are
// widened to fp32 once per block, and y goes back through a buffer.
// Sequences are cut into super-chunks as in the real scan: an aggregate
// pass runs each super-chunk but the last from a zero state and records its
// end state and its sum of steps (in double: the turn w * sum dt of a long
// super-chunk must keep its fractional part), and the main pass enters
// super-chunk j with
//   h <- exp(A sum_k) h + h_k      over k < j.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "scan.cuh"

namespace mamba {

// jobs (warps) per CTA: one, so that the jobs spread evenly over the SMs
// (the mid shape's 1,536 jobs in CTAs of four left 88 SMs with twelve warps
// and 60 with eight; 0.795 -> 0.781 ms)
constexpr int kCplxWarps = 1;
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
  int async;                    // u, delta, y, B and C rows come in 16-byte pieces (cp.async staging)
};

#ifndef MAMBA_CPLX_LANES
#define MAMBA_CPLX_LANES 2  // lanes per channel from 8 states on (1 or 2)
#endif
template <int N>
__host__ __device__ constexpr int cplx_lanes_per_channel() { return N >= 8 ? MAMBA_CPLX_LANES : 1; }
template <int N>
__host__ __device__ constexpr int cplx_channels_per_warp() { return 32 / cplx_lanes_per_channel<N>(); }

template <typename TIO, int N>
struct ComplexSmem {
  static constexpr int kCPW = cplx_channels_per_warp<N>();
  // per warp: [2] raw u and dt [32 tokens][kCPW], [2] raw B and C [32][N],
  // B and C widened [32][N] fp32, y [32][kCPW] fp32
  static constexpr int kRawU = kCplxBlock * kCPW * (int)sizeof(TIO);
  static constexpr int kRawB = kCplxBlock * N * (int)sizeof(TIO);
  static constexpr int kU = 0;
  static constexpr int kDt = kU + 2 * kRawU;
  static constexpr int kBr = kDt + 2 * kRawU;
  static constexpr int kCr = kBr + 2 * kRawB;
  static constexpr int kB = kCr + 2 * kRawB;
  static constexpr int kC = kB + kCplxBlock * N * 4;
  static constexpr int kY = kC + kCplxBlock * N * 4;
  static constexpr int kWarp = kY + kCplxBlock * kCPW * 4;
  static constexpr int kBytes = kCplxWarps * kWarp;
  static_assert(kRawU % 16 == 0 && kRawB % 16 == 0, "16-byte copy destinations");
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
// m = expm1(x) is returned too.
__device__ __forceinline__ void expm1_complex(float x, float v, float* re, float* im, float* m_out = nullptr) {
  const float m = expm1_small(x);
  float s, c;
  sincos_reduced(v, &s, &c);
  const float s2 = 2.0f * s * s;
  *re = fmaf(m, 1.0f - s2, -s2);
  *im = (1.0f + m) * (2.0f * s * c);
  if (m_out) *m_out = m;
}

template <typename TIO, int N, bool AGG>
__global__ void __launch_bounds__(kCplxWarps * 32)
complex_scan_kernel(const ComplexArgs a) {
  using L = ComplexSmem<TIO, N>;
  constexpr int LPC = cplx_lanes_per_channel<N>();  // lanes per channel
  constexpr int CPW = L::kCPW;                      // channels per warp
  constexpr int NH = N / LPC;                       // states per lane
  static_assert(NH % 2 == 0, "states are walked in pairs");
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
  const int cl = lane / LPC;         // channel of this lane within the warp
  const int half = lane % LPC;       // which half of the channel's states
  const int n0 = half * NH;          // first state of this lane
  const int d0 = CPW * g;            // first channel of the warp
  const int d = d0 + cl;
  const bool active = d < a.channels;
  const int dc = active ? d : a.channels - 1;  // inactive lanes read a valid channel, write nothing
  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;
  const float* Are = a.A_re + (int64_t)dc * N;
  const float* Aim = a.A_im + (int64_t)dc * N;

  unsigned char* wsm = cplx_smem + warp * L::kWarp;
  float* sB = reinterpret_cast<float*>(wsm + L::kB);
  float* sC = reinterpret_cast<float*>(wsm + L::kC);
  float* sy = reinterpret_cast<float*>(wsm + L::kY);

  // S4D-Lin structure on every channel of the warp: A[n] = (n+1) a + i n w
  // exactly (fp32), i.e. A[n+1] - A[n] = a + i w for all n
  float sa, sw;  // a and w / 2 of the step a + i w
  bool structured;
  {
    const float a0 = __ldg(Are), w1 = __ldg(Aim + 1);
    bool ok = a0 < 0.0f;
    for (int n = 0; n < N; ++n) ok &= __ldg(Are + n) == (float)(n + 1) * a0 && __ldg(Aim + n) == (float)n * w1;
    structured = __all_sync(0xffffffffu, ok);
    sa = a0;
    sw = 0.5f * w1;
  }
  // the state (this lane's states n0 .. n0 + NH - 1) entering the super-chunk
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
    // h <- exp(A sum_k) h + h_k over the earlier super-chunks
    for (int k = 0; k < j; ++k) {
      const int64_t slot = (b * (a.supers - 1) + k) * a.channels + dc;
      const double sd = a.agg_sd[slot];
      const float2* hk = reinterpret_cast<const float2*>(a.agg_h) + slot * N + n0;
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const float mag = ex2_approx((float)(sd * (double)__ldg(Are + n0 + i)) * 1.4426950408889634f);
        double turn = sd * (double)__ldg(Aim + n0 + i);
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
  const TIO* ug = static_cast<const TIO*>(a.u) + b * a.len * a.channels;
  const TIO* dg = static_cast<const TIO*>(a.delta) + b * a.len * a.channels;
  const TIO* Bg = static_cast<const TIO*>(a.B) + b * a.len * N;
  const TIO* Cg = static_cast<const TIO*>(a.C) + b * a.len * N;
  TIO* yg = static_cast<TIO*>(a.y) + b * a.len * a.channels;
  double sd_total = 0.0;

  // Copy block [t0, t0 + cnt) into buffer `buf`: 16-byte cp.async pieces
  // (zero-filled past the sequence and the last channel) when a.async, else
  // plain loads.  u and dt rows: the warp's CPW channels; B and C: N values.
  constexpr int kPU = CPW * (int)sizeof(TIO) / 16;  // 16-byte pieces of a u row
  constexpr bool kRows16 = (N * (int)sizeof(TIO)) % 16 == 0;  // B rows are whole 16-byte pieces
  constexpr int kPB = kRows16 ? N * (int)sizeof(TIO) / 16 : 1;   // of a B row
  auto issue = [&](int64_t t0, int cnt, int buf) {
    if (kRows16 && a.async) {
      const uint32_t su0 = smem_addr(wsm + L::kU + buf * L::kRawU);
      const uint32_t sd0 = smem_addr(wsm + L::kDt + buf * L::kRawU);
      for (int i = lane; i < kCplxBlock * kPU; i += 32) {
        const int k = i / kPU, q = i % kPU;
        const int ch = d0 + q * (16 / (int)sizeof(TIO));
        const bool in = k < cnt && ch < a.channels;
        const int64_t off = in ? (t0 + k) * a.channels + ch : 0;
        cp_async16_zfill(su0 + i * 16, ug + off, in);
        cp_async16_zfill(sd0 + i * 16, dg + off, in);
      }
      const uint32_t sb0 = smem_addr(wsm + L::kBr + buf * L::kRawB);
      const uint32_t sc0 = smem_addr(wsm + L::kCr + buf * L::kRawB);
      for (int i = lane; i < kCplxBlock * kPB; i += 32) {
        const int k = i / kPB, q = i % kPB;
        const bool in = k < cnt;
        const int64_t off = in ? (t0 + k) * N + q * (16 / (int)sizeof(TIO)) : 0;
        cp_async16_zfill(sb0 + i * 16, Bg + off, in);
        if (!AGG) cp_async16_zfill(sc0 + i * 16, Cg + off, in);
      }
    } else {
      TIO* u0 = reinterpret_cast<TIO*>(wsm + L::kU + buf * L::kRawU);
      TIO* dt0 = reinterpret_cast<TIO*>(wsm + L::kDt + buf * L::kRawU);
      for (int i = lane; i < kCplxBlock * CPW; i += 32) {
        const int k = i / CPW, c = i % CPW;
        const bool in = k < cnt && d0 + c < a.channels;
        u0[i] = in ? ug[(t0 + k) * a.channels + d0 + c] : from_f32<TIO>(0.0f);
        dt0[i] = in ? dg[(t0 + k) * a.channels + d0 + c] : from_f32<TIO>(0.0f);
      }
      TIO* b0 = reinterpret_cast<TIO*>(wsm + L::kBr + buf * L::kRawB);
      TIO* c0 = reinterpret_cast<TIO*>(wsm + L::kCr + buf * L::kRawB);
      for (int i = lane; i < kCplxBlock * N; i += 32) {
        const int k = i / N;
        b0[i] = k < cnt ? Bg[t0 * N + i] : from_f32<TIO>(0.0f);
        if (!AGG) c0[i] = k < cnt ? Cg[t0 * N + i] : from_f32<TIO>(0.0f);
      }
    }
    cp_async_commit();  // (an empty group without copies)
  };
  // the block in `buf` has landed: widen its B and C rows to fp32
  auto widen = [&](int buf) {
    const TIO* b0 = reinterpret_cast<const TIO*>(wsm + L::kBr + buf * L::kRawB);
    const TIO* c0 = reinterpret_cast<const TIO*>(wsm + L::kCr + buf * L::kRawB);
#pragma unroll 4
    for (int i = lane; i < kCplxBlock * N; i += 32) {
      sB[i] = to_f32(b0[i]);
      if (!AGG) sC[i] = to_f32(c0[i]);
    }
    __syncwarp();
  };
  // y of the block from sy to global memory (16-byte stores when a.async)
  auto flush = [&](int64_t t0, int cnt) {
    if (AGG) return;
    __syncwarp();
    if (a.async) {
      constexpr int kE = 16 / (int)sizeof(TIO);  // elements per 16-byte piece
      for (int i = lane; i < kCplxBlock * kPU; i += 32) {
        const int k = i / kPU, q = i % kPU;
        const int ch = d0 + q * kE;
        if (k < cnt && ch < a.channels) {
          TIO v[kE];
#pragma unroll
          for (int e = 0; e < kE; ++e) v[e] = from_f32<TIO>(sy[k * CPW + q * kE + e]);
          *reinterpret_cast<uint4*>(yg + (t0 + k) * a.channels + ch) = *reinterpret_cast<const uint4*>(v);
        }
      }
    } else {
      for (int i = lane; i < kCplxBlock * CPW; i += 32) {
        const int k = i / CPW, c = i % CPW;
        if (k < cnt && d0 + c < a.channels) yg[(t0 + k) * a.channels + d0 + c] = from_f32<TIO>(sy[i]);
      }
    }
  };
  // y of token k of the block, summed over the lanes of the channel
  auto emit = [&](int k, float x, float acc) {
    if (LPC == 2) acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) sy[k * CPW + cl] = fmaf(Dd, x, acc);
  };
  // walk the super-chunk: block i computes while block i + 1 is copied
  auto run = [&](auto&& token) {
    const int nblk = (int)((t_end - t_begin + kCplxBlock - 1) / kCplxBlock);
    if (nblk > 0) issue(t_begin, (int)(t_end - t_begin < kCplxBlock ? t_end - t_begin : kCplxBlock), 0);
    for (int bi = 0; bi < nblk; ++bi) {
      const int64_t t0 = t_begin + (int64_t)bi * kCplxBlock;
      const int cnt = t_end - t0 < kCplxBlock ? (int)(t_end - t0) : kCplxBlock;
      const int buf = bi & 1;
      __syncwarp();  // every lane is done with the buffer the next copies overwrite
      if (bi + 1 < nblk) {
        const int64_t t1 = t0 + kCplxBlock;
        issue(t1, t_end - t1 < kCplxBlock ? (int)(t_end - t1) : kCplxBlock, buf ^ 1);
      } else {
        cp_async_commit();
      }
      cp_async_wait<1>();  // block bi has landed (this lane's copies) ...
      __syncwarp();        // ... and every lane's
      widen(buf);
      const TIO* u0 = reinterpret_cast<const TIO*>(wsm + L::kU + buf * L::kRawU);
      const TIO* dt0 = reinterpret_cast<const TIO*>(wsm + L::kDt + buf * L::kRawU);
      if (cnt == kCplxBlock) {
#pragma unroll 2
        for (int k = 0; k < kCplxBlock; ++k) token(k, u0, dt0);
      } else {
        for (int k = 0; k < cnt; ++k) token(k, u0, dt0);
      }
      flush(t0, cnt);
    }
    cp_async_wait<0>();
  };

  if (structured) {
    // pairs of states: 1/A = ir - i ni (so Re(g / A) = gr ir + gi ni) and
    // the scaled state g = A h
    float2 ir2[NH / 2], ni2[NH / 2], gr2[NH / 2], gi2[NH / 2];
#pragma unroll
    for (int p = 0; p < NH / 2; ++p) {
      float irv[2], niv[2], grv[2], giv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * p + e;
        const float re = __ldg(Are + n0 + i), im = __ldg(Aim + n0 + i);
        const float inv = 1.0f / fmaf(re, re, im * im);
        irv[e] = re * inv;
        niv[e] = im * inv;
        grv[e] = fmaf(re, hr[i], -im * hi[i]);
        giv[e] = fmaf(re, hi[i], im * hr[i]);
      }
      ir2[p] = make_float2(irv[0], irv[1]);
      ni2[p] = make_float2(niv[0], niv[1]);
      gr2[p] = make_float2(grv[0], grv[1]);
      gi2[p] = make_float2(giv[0], giv[1]);
    }
    // One token.  The decays of the lane's states come from a product chain
    // of pair steps from (E_n0, E_n0+1): E_n0+1 = E_n0 + F + E_n0 F, then
    // E <- E + F2 + E F2 (F2 = F (2 + F)).  The exponential's inputs per
    // lane: (a, w/2) for the first lane of a channel, ((n0+1) a, n0 w/2) for
    // the second.
    const float xa = half ? (float)(n0 + 1) * sa : sa, xw = half ? (float)n0 * sw : sw;
    auto token = [&](int k, const TIO* u0, const TIO* dt0) {
      const float x = to_f32(u0[k * CPW + cl]);
      const float dt = to_f32(dt0[k * CPW + cl]);
      if (AGG) sd_total += (double)dt;
      // one complex exponential per lane: the first lane of a channel takes
      // F = exp(dt (a + i w)) - 1 (and m = expm1(dt a) = E_0), the second
      // E_{n0} = exp(dt A_{n0}) - 1 directly (A_{n0} = (n0+1) a + i n0 w) and
      // F from its partner
      float fr, fi, m;
      expm1_complex(dt * xa, dt * xw, &fr, &fi, &m);
      float e1r = m, e1i = 0.0f;  // the lane's first state's E
      if constexpr (LPC == 2) {
        const float pr = __shfl_xor_sync(0xffffffffu, fr, 1), pi = __shfl_xor_sync(0xffffffffu, fi, 1);
        if (half) {
          e1r = fr;
          e1i = fi;
          fr = pr;
          fi = pi;
        }
      }
      const float f2r = fmaf(fr, 2.0f + fr, -fi * fi);
      const float f2i = fi * fmaf(2.0f, fr, 2.0f);
      auto step = [](float2& er, float2& ei, float2 gr, float2 gi, float2 ngi) {
        const float2 nr = __ffma2_rn(ei, ngi, __ffma2_rn(er, gr, __fadd2_rn(er, gr)));
        const float2 ni = __ffma2_rn(ei, gr, __ffma2_rn(er, gi, __fadd2_rn(ei, gi)));
        er = nr;
        ei = ni;
      };
      // (E_n0, E_n0+1), E_n0+1 = E_n0 + F + E_n0 F
      float2 er = make_float2(e1r, e1r + fr + fmaf(e1r, fr, -e1i * fi));
      float2 ei = make_float2(e1i, e1i + fi + fmaf(e1r, fi, e1i * fr));
      const float2 Fr = make_float2(f2r, f2r), Fi = make_float2(f2i, f2i), nFi = make_float2(-f2i, -f2i);
      const float2 x2 = make_float2(x, x);
      const float4* Bt = reinterpret_cast<const float4*>(sB + k * N + n0);
      const float4* Ct = reinterpret_cast<const float4*>(sC + k * N + n0);
      float2 accA = make_float2(0.0f, 0.0f), accB = make_float2(0.0f, 0.0f);
      // g <- g + E v, v = g + B x (B x real):
      //   Re: gr + er vr - ei gi,   Im: gi + er gi + ei vr
      auto update = [&](int p, float2 bb, float2 cc, float2& acc) {
        const float2 vr = __ffma2_rn(bb, x2, gr2[p]);
        const float2 nei = make_float2(-ei.x, -ei.y);
        const float2 tr = __ffma2_rn(nei, gi2[p], __ffma2_rn(er, vr, gr2[p]));
        const float2 ti = __ffma2_rn(ei, vr, __ffma2_rn(er, gi2[p], gi2[p]));
        gr2[p] = tr;
        gi2[p] = ti;
        if (!AGG) acc = __ffma2_rn(cc, __ffma2_rn(ti, ni2[p], __fmul2_rn(tr, ir2[p])), acc);
      };
#pragma unroll
      for (int p2 = 0; p2 < NH / 4; ++p2) {  // two pairs per 16-byte B / C read
        const float4 bq = Bt[p2];
        const float4 cq = AGG ? make_float4(0.f, 0.f, 0.f, 0.f) : Ct[p2];
        if (p2 > 0) step(er, ei, Fr, Fi, nFi);
        update(2 * p2, make_float2(bq.x, bq.y), make_float2(cq.x, cq.y), accA);
        step(er, ei, Fr, Fi, nFi);
        update(2 * p2 + 1, make_float2(bq.z, bq.w), make_float2(cq.z, cq.w), accB);
      }
      if (!AGG) emit(k, x, (accA.x + accA.y) + (accB.x + accB.y));
    };
    run(token);
    // back to h = g / A = (gr ir + gi ni) + i (gi ir - gr ni)
#pragma unroll
    for (int p = 0; p < NH / 2; ++p) {
      hr[2 * p] = fmaf(gr2[p].x, ir2[p].x, gi2[p].x * ni2[p].x);
      hi[2 * p] = fmaf(gi2[p].x, ir2[p].x, -gr2[p].x * ni2[p].x);
      hr[2 * p + 1] = fmaf(gr2[p].y, ir2[p].y, gi2[p].y * ni2[p].y);
      hi[2 * p + 1] = fmaf(gi2[p].y, ir2[p].y, -gr2[p].y * ni2[p].y);
    }
  } else {
    // general A: one complex exponential per state; per state a, w / 2 and
    // 1/A = conj(A) / |A|^2
    float ar[NH], wh[NH], iar[NH], iai[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const float re = __ldg(Are + n0 + i), im = __ldg(Aim + n0 + i);
      const float inv = 1.0f / fmaf(re, re, im * im);
      ar[i] = re;
      wh[i] = 0.5f * im;
      iar[i] = re * inv;
      iai[i] = -im * inv;
    }
    auto token = [&](int k, const TIO* u0, const TIO* dt0) {
      const float x = to_f32(u0[k * CPW + cl]);
      const float dt = to_f32(dt0[k * CPW + cl]);
      if (AGG) sd_total += (double)dt;
      const float* Bt = sB + k * N + n0;
      const float* Ct = sC + k * N + n0;
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        float er, ei;
        expm1_complex(dt * ar[i], dt * wh[i], &er, &ei);  // exp(dt A) - 1
        const float bx = Bt[i] * x;
        const float gr = fmaf(er, iar[i], -ei * iai[i]) * bx;  // Re((E / A) B x)
        const float gi = fmaf(er, iai[i], ei * iar[i]) * bx;   // Im((E / A) B x)
        const float nr = hr[i] + fmaf(er, hr[i], fmaf(-ei, hi[i], gr));
        const float ni = hi[i] + fmaf(er, hi[i], fmaf(ei, hr[i], gi));
        hr[i] = nr;
        hi[i] = ni;
        if (!AGG) acc = fmaf(Ct[i], nr, acc);
      }
      if (!AGG) emit(k, x, acc);
    };
    run(token);
  }

  griddep_launch_dependents();
  if (!active) return;
  if (AGG) {
    const int64_t slot = (b * (a.supers - 1) + j) * a.channels + d;
    if (half == 0) a.agg_sd[slot] = sd_total;
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
