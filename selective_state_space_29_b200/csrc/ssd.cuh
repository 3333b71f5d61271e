// ssd.cuh -- Mamba-2's restricted scan (one scalar A per head, one step per
// (token, head)) in its chunked matrix form, on the tensor cores.
//
// With A = a_h * I the decay from token s to token t is the same scalar for
// every state and channel of head h, so within a chunk of Q tokens
//   y_t = e^{a(cum_t)} C_t . S_in  +  sum_{s<=t} (C_t . B_s) e^{a(cum_t - cum_s)} w_s x_s
//   S_out = e^{a(cum_end)} S_in + sum_s e^{a(cum_end - cum_s)} w_s B_s x_s^T
// ("Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)", "Mamba-2 ve
// Güncel Gelişmeler": the SSM equals a masked attention-like form; the
// Mamba-3 page, "Karmaşık Değerli Durum Güncellemesi": Mamba-2's scalar
// transition).  cum is the running sum of the steps inside the chunk and w_s
// the input weight of the discretisation: (e^{a dt} - 1)/a for the
// zero-order hold, dt for exponential Euler.
//
// A CTA of four warps owns one (batch row, head, super-chunk) and walks its
// chunks of 64 tokens in order; warp w owns the chunk's rows 16w..16w+15.
// Per chunk (mma.sync m16n8k16, bf16 operands, fp32 accumulators):
//   Y   = C S_in                         [16 x 64] += [16 x N][N x 64]
//   Y  *= e^{a cum_t} (per row)
//   G   = C B^T                          [16 x 16(k+1)], causal blocks only
//   M   = G o e^{a(cum_t - cum_s)} o w_s (masked s > t), rounded to bf16 in
//         registers: the accumulator fragment is the next MMA's A fragment
//   Y  += M X                            [16 x 64] += [16 x 16(w+1)][.. x 64]
//   y   = Y + D x  -> bf16 -> shared -> 16-byte stores
//   dS  = Bw^T X, Bw_s = e^{a(cum_end - cum_s)} w_s B_s     (warp w: 16 channels)
//   S   = e^{a cum_end} S + dS           (fp32 registers; a bf16 copy in
//                                          shared memory feeds the next Y_off)
// x, B and C stream through a 3-stage cp.async ring (16-byte copies,
// XOR-swizzled rows so that every ldmatrix is free of bank conflicts).
//
// Long sequences with few (batch, head) pairs are cut into super-chunks: an
// aggregate kernel runs each super-chunk but the last from a zero state and
// records its end state and total decay; the main kernel folds the
// aggregates of the earlier super-chunks into its entering state.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"

namespace mamba {

constexpr int kSsdQ = 64;       // tokens per chunk
constexpr int kSsdP = 64;       // channels per head
constexpr int kSsdWarps = 4;    // warp w owns chunk rows 16w..16w+15
constexpr int kSsdStages = 3;   // cp.async ring depth (chunks in flight)

struct SsdArgs {
  const __nv_bfloat16* x;       // (batch, len, heads*64)
  const __nv_bfloat16* dt;      // (batch, len, heads)
  const float* A;               // (heads)
  const __nv_bfloat16* B;       // (batch, len, N)
  const __nv_bfloat16* C;       // (batch, len, N)
  const float* D;               // (heads*64) or null
  const float* h0;              // (batch, heads*64, N) or null
  __nv_bfloat16* y;             // (batch, len, heads*64)
  float* final_state;           // (batch, heads*64, N) or null
  float* agg_state;             // (batch*heads, supers-1, 64, N): super-chunk end state from zero
  float* agg_decay;             // (batch*heads, supers-1): log2 of its total decay
  int64_t len;
  int heads;
  int supers;                   // super-chunks per (batch row, head)
  int64_t super_len;            // tokens per super-chunk, a multiple of 64
  int euler;                    // input weight dt (exponential Euler) instead of the ZOH weight
};

// Byte offset of 16-byte chunk `ch` of row `row` in a tile whose rows are R
// chunks long: the chunk index is XORed with the row's position among the
// rows that share a 128-byte line, so that 8 consecutive rows at one chunk
// column fall in 8 different bank groups.
template <int R>
__device__ __forceinline__ uint32_t ssd_swz(int row, int ch) {
  constexpr int kRowsPerLine = 8 / R;
  return (uint32_t)(row * R * 16 + ((ch ^ ((row / kRowsPerLine) & (R - 1))) * 16));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0: nothing is read, the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// D[16x8] += A[16x16] B[16x8], bf16 in, fp32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int N>
struct SsdSmem {
  static constexpr int R = N / 8;                  // 16-byte chunks per B / C row
  static constexpr int kX = kSsdQ * kSsdP * 2;     // one x tile
  static constexpr int kBC = kSsdQ * N * 2;        // one B or C tile
  static constexpr int kStage = kX + 2 * kBC;
  static constexpr int kRing = kSsdStages * kStage;
  static constexpr int kBw = kRing;                // [64 tokens][N] bf16
  static constexpr int kS = kBw + kBC;             // [64 channels][N] bf16 copy of the state
  static constexpr int kY = kS + kSsdP * N * 2;    // [64][64] bf16 output staging
  static constexpr int kCum = kY + kSsdQ * kSsdP * 2;  // per warp: cum (log2) and w for 64 tokens
  static constexpr int kBytes = kCum + kSsdWarps * 2 * kSsdQ * 4;
  // CTAs per SM the register budget is set for (shared memory allows 4 at
  // 16 states, 3 at 32, 2 at 64)
  static constexpr int kMinBlocks = N == 16 ? 4 : 2;
};

template <int N, bool AGG>
__global__ void __launch_bounds__(kSsdWarps * 32, SsdSmem<N>::kMinBlocks)
ssd_chunk_kernel(const SsdArgs a) {
  using L = SsdSmem<N>;
  constexpr int R = L::R;
  constexpr int KS = N / 16;   // k-steps over states
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int64_t channels = (int64_t)a.heads * kSsdP;

  // job: (batch row, head, super-chunk); the aggregate kernel has one
  // super-chunk fewer per (batch row, head)
  const int per_seq = AGG ? a.supers - 1 : a.supers;
  const int64_t seq = blockIdx.x / per_seq;
  const int j = (int)(blockIdx.x % per_seq);
  const int64_t b = seq / a.heads;
  const int h = (int)(seq % a.heads);
  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;
  const int nchunks = (int)((t_end - t_begin + kSsdQ - 1) / kSsdQ);

  griddep_wait();  // inputs (and the aggregates) may come from the previous kernel

  const float a_h = __ldg(a.A + h);
  const float a2 = a_h * 1.4426950408889634f;  // a in log2 units
  const __nv_bfloat16* xg = a.x + (b * a.len) * channels + (int64_t)h * kSsdP;
  const __nv_bfloat16* Bg = a.B + (b * a.len) * N;
  const __nv_bfloat16* Cg = a.C + (b * a.len) * N;
  const unsigned short* dtg = reinterpret_cast<const unsigned short*>(a.dt) + (b * a.len) * a.heads + h;

  // stage one chunk's x, B (and C) into ring slot `slot`
  auto load_chunk = [&](int c, int slot) {
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    const uint32_t sx = sbase + slot * L::kStage;
#pragma unroll
    for (int i = tid; i < kSsdQ * 8; i += kSsdWarps * 32) {
      const int row = i >> 3, ch = i & 7;
      const bool ok = t0 + row < t_end;
      cp_async16(sx + ssd_swz<8>(row, ch), ok ? (const void*)(xg + (t0 + row) * channels + ch * 8) : (const void*)a.x,
                 ok);
    }
    const uint32_t sb = sx + L::kX;
#pragma unroll
    for (int i = tid; i < kSsdQ * R; i += kSsdWarps * 32) {
      const int row = i / R, ch = i % R;
      const bool ok = t0 + row < t_end;
      cp_async16(sb + ssd_swz<R>(row, ch), ok ? (const void*)(Bg + (t0 + row) * N + ch * 8) : (const void*)a.B, ok);
      if (!AGG)
        cp_async16(sb + L::kBC + ssd_swz<R>(row, ch),
                   ok ? (const void*)(Cg + (t0 + row) * N + ch * 8) : (const void*)a.C, ok);
    }
  };
  auto load_dt = [&](int c, int k) -> float {
    const int64_t t = t_begin + (int64_t)c * kSsdQ + k;
    if (c >= nchunks || t >= t_end) return 0.0f;  // padding tokens: no decay, no input
    return __uint_as_float((uint32_t)__ldg(dtg + t * a.heads) << 16);
  };

  // the state: warp w holds channels 16w..16w+15 for all N states, in the
  // accumulator layout of dS (row = state, column = channel)
  float S[KS][2][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int e = 0; e < 4; ++e) S[mt][jj][e] = 0.0f;
  auto s_index = [&](int mt, int jj, int e, int* n, int* p) {
    *n = 16 * mt + g + 8 * (e >> 1);
    *p = 16 * warp + 8 * jj + 2 * q + (e & 1);
  };
  if (!AGG) {
    if (a.h0) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            int n, p;
            s_index(mt, jj, e, &n, &p);
            S[mt][jj][e] = __ldg(a.h0 + ((b * a.heads + h) * kSsdP + p) * N + n);
          }
    }
    // fold in the super-chunks before this one
    for (int k = 0; k < j; ++k) {
      const int64_t agg = seq * (a.supers - 1) + k;
      const float dec = exp2f(__ldg(a.agg_decay + agg));
      const float* as = a.agg_state + agg * (kSsdP * N);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            int n, p;
            s_index(mt, jj, e, &n, &p);
            S[mt][jj][e] = fmaf(dec, S[mt][jj][e], __ldg(as + p * N + n));
          }
    }
  }
  // bf16 copy of the state for the next chunk's C S_in (state n, channel p)
  auto store_state_copy = [&]() {
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int n, p;
          s_index(mt, jj, e, &n, &p);
          const __nv_bfloat16 v = __float2bfloat16_rn(S[mt][jj][e]);
          *reinterpret_cast<__nv_bfloat16*>(smem + L::kS + ssd_swz<R>(p, n >> 3) + (n & 7) * 2) = v;
        }
  };
  if (!AGG) store_state_copy();

  float* cum_w = reinterpret_cast<float*>(smem + L::kCum) + warp * 2 * kSsdQ;  // [64] cum (log2), [64] w
  float* wt_w = cum_w + kSsdQ;
  float total_log2 = 0.0f;

  // prologue: the first kSsdStages-1 chunks
#pragma unroll
  for (int s = 0; s < kSsdStages - 1; ++s) {
    if (s < nchunks) load_chunk(s, s);
    cp_async_commit();
  }
  float dt0 = load_dt(0, lane), dt1 = load_dt(0, lane + 32);

  for (int c = 0; c < nchunks; ++c) {
    const int slot = c % kSsdStages;
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    // next chunk's steps, one chunk ahead
    const float ndt0 = load_dt(c + 1, lane), ndt1 = load_dt(c + 1, lane + 32);

    // running log2 decay inside the chunk (every warp computes its own copy)
    float v0 = dt0 * a2, v1 = dt1 * a2;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float n0 = __shfl_up_sync(0xffffffffu, v0, o);
      const float n1 = __shfl_up_sync(0xffffffffu, v1, o);
      if (lane >= o) {
        v0 += n0;
        v1 += n1;
      }
    }
    v1 += __shfl_sync(0xffffffffu, v0, 31);
    const float cum_end = __shfl_sync(0xffffffffu, v1, 31);
    total_log2 += cum_end;
    const float w0 = a.euler ? dt0 : expm1f(dt0 * a_h) / a_h;
    const float w1 = a.euler ? dt1 : expm1f(dt1 * a_h) / a_h;
    __syncwarp();
    cum_w[lane] = v0;
    cum_w[lane + 32] = v1;
    wt_w[lane] = w0;
    wt_w[lane + 32] = w1;
    __syncwarp();

    cp_async_wait<kSsdStages - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();                  // everyone's; and chunk c-1 is done with its slot
    if (c + kSsdStages - 1 < nchunks) load_chunk(c + kSsdStages - 1, (c + kSsdStages - 1) % kSsdStages);
    cp_async_commit();

    const uint32_t sx = sbase + slot * L::kStage;
    const uint32_t sb = sx + L::kX;
    const uint32_t sc = sb + L::kBC;

    // Bw rows of this warp's 16 tokens: e^{a(cum_end - cum_s)} w_s B_s
    {
      constexpr int kPer = 16 * N / 32;  // elements per lane
      const int row = 16 * warp + lane / (32 / 16);
      static_assert(kPer % 2 == 0, "pairs");
      const int n0 = (lane % 2) * kPer;
      const float f = ex2_approx(cum_end - cum_w[row]) * wt_w[row];
#pragma unroll
      for (int i = 0; i < kPer; i += 2) {
        const int n = n0 + i;
        const uint32_t off = ssd_swz<R>(row, n >> 3) + (n & 7) * 2;
        const __nv_bfloat162 bv = *reinterpret_cast<const __nv_bfloat162*>(smem + (sb - sbase) + off);
        const float2 bf = __bfloat1622float2(bv);
        *reinterpret_cast<uint32_t*>(smem + L::kBw + off) = pack_bf16(bf.x * f, bf.y * f);
      }
    }

    if (!AGG) {
      const int r0 = 16 * warp + g, r1 = r0 + 8;
      const float cr0 = cum_w[r0], cr1 = cum_w[r1];
      // C fragments of this warp's rows (A operand, row-major [t][n])
      uint32_t cf[KS][4];
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        ldsm_x4(cf[kk], sc + ssd_swz<R>(16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * kk + (lane >> 4)));

      // Y = e^{a cum_t} C S_in
      float Y[8][4];
#pragma unroll
      for (int jt = 0; jt < 8; ++jt)
#pragma unroll
        for (int e = 0; e < 4; ++e) Y[jt][e] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {
          uint32_t sf[4];
          ldsm_x4(sf, sbase + L::kS + ssd_swz<R>(16 * jp + (lane & 7) + 8 * (lane >> 4), 2 * kk + ((lane >> 3) & 1)));
          mma_bf16(Y[2 * jp], cf[kk], sf[0], sf[1]);
          mma_bf16(Y[2 * jp + 1], cf[kk], sf[2], sf[3]);
        }
      {
        const float e0 = ex2_approx(cr0), e1 = ex2_approx(cr1);
#pragma unroll
        for (int jt = 0; jt < 8; ++jt) {
          Y[jt][0] *= e0;
          Y[jt][1] *= e0;
          Y[jt][2] *= e1;
          Y[jt][3] *= e1;
        }
      }

      // causal part, one 16-token column block at a time
#pragma unroll
      for (int ks = 0; ks < kSsdWarps; ++ks) {
        if (ks <= warp) {
          // G for columns 16ks..16ks+15 (two n-tiles)
          float G[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            uint32_t bf[4];
            ldsm_x4(bf, sb + ssd_swz<R>(16 * ks + (lane & 7) + 8 * (lane >> 4), 2 * kk + ((lane >> 3) & 1)));
            mma_bf16(G[0], cf[kk], bf[0], bf[1]);
            mma_bf16(G[1], cf[kk], bf[2], bf[3]);
          }
          // M = G o e^{a(cum_t - cum_s)} o w_s, zero above the diagonal
          uint32_t am[4];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int s0 = 16 * ks + 8 * half + 2 * q;
            const float2 cs = *reinterpret_cast<const float2*>(cum_w + s0);
            const float2 ws = *reinterpret_cast<const float2*>(wt_w + s0);
            const float x00 = s0 <= r0 ? cr0 - cs.x : -INFINITY;
            const float x01 = s0 + 1 <= r0 ? cr0 - cs.y : -INFINITY;
            const float x10 = s0 <= r1 ? cr1 - cs.x : -INFINITY;
            const float x11 = s0 + 1 <= r1 ? cr1 - cs.y : -INFINITY;
            am[2 * half + 0] = pack_bf16(G[half][0] * ex2_approx(x00) * ws.x, G[half][1] * ex2_approx(x01) * ws.y);
            am[2 * half + 1] = pack_bf16(G[half][2] * ex2_approx(x10) * ws.x, G[half][3] * ex2_approx(x11) * ws.y);
          }
          // Y += M X for tokens 16ks..16ks+15
#pragma unroll
          for (int jp = 0; jp < 4; ++jp) {
            uint32_t xf[4];
            ldsm_x4_t(xf, sx + ssd_swz<8>(16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * jp + (lane >> 4)));
            mma_bf16(Y[2 * jp], am, xf[0], xf[1]);
            mma_bf16(Y[2 * jp + 1], am, xf[2], xf[3]);
          }
        }
      }

      // y = Y + D x -> bf16, staged per warp, then 16-byte row stores
      const float* Dh = a.D ? a.D + (int64_t)h * kSsdP : nullptr;
#pragma unroll
      for (int jt = 0; jt < 8; ++jt) {
        const int p = 8 * jt + 2 * q;
        const float2 dd = Dh ? __ldg(reinterpret_cast<const float2*>(Dh + p)) : make_float2(0.f, 0.f);
        const uint32_t o0 = ssd_swz<8>(r0, jt) + 4 * q, o1 = ssd_swz<8>(r1, jt) + 4 * q;
        const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(smem + (sx - sbase) + o0));
        const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(smem + (sx - sbase) + o1));
        *reinterpret_cast<uint32_t*>(smem + L::kY + o0) =
            pack_bf16(fmaf(dd.x, x0.x, Y[jt][0]), fmaf(dd.y, x0.y, Y[jt][1]));
        *reinterpret_cast<uint32_t*>(smem + L::kY + o1) =
            pack_bf16(fmaf(dd.x, x1.x, Y[jt][2]), fmaf(dd.y, x1.y, Y[jt][3]));
      }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = lane + 32 * k;
        const int row = 16 * warp + (i >> 3), ch = i & 7;
        if (t0 + row < t_end) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + L::kY + ssd_swz<8>(row, ch));
          *reinterpret_cast<uint4*>(a.y + (b * a.len + t0 + row) * channels + (int64_t)h * kSsdP + ch * 8) = v;
        }
      }
    }

    __syncthreads();  // Bw complete; every read of the state copy is done

    // dS = Bw^T X for channels 16w..16w+15, then S = e^{a cum_end} S + dS
    {
      float dS[KS][2][4];
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) dS[mt][jj][e] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < kSsdQ / 16; ++ks) {
        uint32_t xf[4];
        ldsm_x4_t(xf, sx + ssd_swz<8>(16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * warp + (lane >> 4)));
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          uint32_t bw[4];
          ldsm_x4_t(bw, sbase + L::kBw + ssd_swz<R>(16 * ks + (lane & 7) + 8 * (lane >> 4), 2 * mt + ((lane >> 3) & 1)));
          mma_bf16(dS[mt][0], bw, xf[0], xf[1]);
          mma_bf16(dS[mt][1], bw, xf[2], xf[3]);
        }
      }
      const float dec = ex2_approx(cum_end);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) S[mt][jj][e] = fmaf(dec, S[mt][jj][e], dS[mt][jj][e]);
    }
    if (!AGG) store_state_copy();
    dt0 = ndt0;
    dt1 = ndt1;
  }
  cp_async_wait<0>();

  griddep_launch_dependents();
  if (AGG) {
    const int64_t agg = seq * (a.supers - 1) + j;
    float* as = a.agg_state + agg * (kSsdP * N);
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int n, p;
          s_index(mt, jj, e, &n, &p);
          as[p * N + n] = S[mt][jj][e];
        }
    if (tid == 0) a.agg_decay[agg] = total_log2;
  } else if (a.final_state && j == a.supers - 1) {
    float* fs = a.final_state + (b * a.heads + h) * (int64_t)(kSsdP * N);
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int n, p;
          s_index(mt, jj, e, &n, &p);
          fs[p * N + n] = S[mt][jj][e];
        }
  }
}

}  // namespace mamba
