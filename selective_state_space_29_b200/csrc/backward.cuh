// backward.cuh -- gradients of the zero-order-hold selective scan (training).
//
// The pages imply training (page "Mamba SSM Nedir? Transformer Alternatifi
// Rehberi (2026)", section "Mamba'nın Yeniliği: Selective SSM": Delta, B and C
// are learned projections of the input) but print no gradient.  This is
// reverse-mode differentiation of the recurrence of section "Ayrık Zamana
// Geçiş".  Per state n and token t, with z = Delta_t A_n, r = exp(z),
// q = r - 1, lam = dL/dh_t (the adjoint):
//     lam_t      = C_t dy_t + r_{t+1} lam_{t+1}          (+ d h_final at the end)
//     du_t       = sum_n lam_t (q / A_n) B_{t,n} + D dy_t
//     dDelta_t   = sum_n lam_t r (A_n h_{t-1} + B_{t,n} x_t)
//     dA_n      += lam_t (Delta_t r h_{t-1} + B_{t,n} x_t Delta_t^2 psi(z)),
//                  psi(z) = (z e^z - (e^z - 1)) / z^2
//     dB_{t,n}  += lam_t x_t q / A_n                      (summed over channels)
//     dC_{t,n}  += dy_t h_t                               (summed over channels)
//     dD        += dy_t x_t,        dh0 = r_0 lam_0
//
// (the dA term is d h_t / d A_n at fixed Delta; psi is evaluated by its
// series where the closed form would cancel, see psi_f).  With
// structured A (A[d,n] = (n+1) A[d,0]) the decays come from one exponential
// per token and the forward kernel's decay chain.
//
// Work decomposition: a warp takes a (batch row, 32-channel group) stream at
// a time, a lane per channel, and walks its tokens in reverse.  The states
// are recomputed tile by tile: the forward kernel leaves the state before
// every tile of T tokens in a checkpoint array; the warp takes a tile in
// two halves, the later first: it re-runs the tile forward from its
// checkpoint through the half's end, writing the half's states h_t to a
// per-warp scratch area ([T/2 + 1][32][N], 64 bytes per lane and token at
// N = 16, read back one token ahead of use; about 78 MB over the resident
// warps, so it stays in L2), then walks the half in reverse.  dB and dC are a reduce-scatter
// (lane i ends with the sum of value i) and one atomic add per lane.  When
// rows are 16-byte aligned, the warp first copies the tile's u, Delta and
// dy rows and its B, C rows into its shared memory (one round of 16-byte
// cp.async copies), so both passes over the tile read shared memory
// instead of waiting on a global load per token.
#pragma once

#include "common.cuh"
#include "scan.cuh"  // expm1_small

namespace mamba {

template <typename TIO>
struct BwdArgs {
  const TIO* u;
  const TIO* delta;
  const float* A;
  const TIO* B;
  const TIO* C;
  const float* D;          // nullable
  const TIO* dy;
  const float* dh_final;   // nullable
  const float* ckpt;       // [batch][ntiles][channels][N]
  float* scratch;          // [warps of the grid][T][32][N]
  TIO* du;
  TIO* ddelta;
  float* dA;               // [channels][N], accumulated (zeroed by the host)
  float* dB;               // [batch][len][N], accumulated
  float* dC;               // [batch][len][N], accumulated
  float* dD;               // [channels] or nullptr, accumulated
  float* dh0;              // [batch][channels][N] or nullptr
  int64_t batch, len, channels;
  int groups_d;            // ceil(channels / 32)
  int tile;                // checkpoint spacing T
  int vec_rows;            // B and C rows may be read with 16-byte vector loads
  int supers;              // S: the sequence is cut into S super-chunks of super_tiles tiles
  int super_tiles;
  float* agg_mu;           // [S][streams][32][N] outgoing adjoint of super-chunk j from zero
  float* agg_sd;           // [S][streams][32] sum of Delta over super-chunk j
  int staged;              // tiles are staged in shared memory (rows 16-byte aligned)
};

// Bytes of one warp's staged tile: u, Delta and dy rows of 32 channels, then
// the B and C rows, for T tokens.
template <typename TIO, int NS>
__host__ __device__ constexpr int bwd_stage_bytes(int T) {
  return (3 * 32 + 2 * NS) * T * (int)sizeof(TIO);
}

// 16-byte asynchronous copy of which the first `bytes` (0..16) come from src
// and the rest is zero-filled
__device__ __forceinline__ void bwd_cp_async(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}

// Stage `rows` token rows of the 32 channels from ch_base on (one row is
// 32 elements, 16-byte pieces; pieces past the last channel are zero-filled)
// to dst, [rows][32]: row r of token t0 + r.  The channel count is a multiple
// of the elements in a piece and the rows are 16-byte aligned on this path.
template <typename TIO>
__device__ __forceinline__ void bwd_stage_rows(uint32_t dst, const TIO* src, int64_t tok0, int rows,
                                               int64_t ch_base, int64_t channels, int lane) {
  constexpr int P = 32 * (int)sizeof(TIO) / 16;  // pieces per row
  constexpr int EPP = 16 / (int)sizeof(TIO);      // channels per piece
  for (int i = lane; i < rows * P; i += 32) {
    const int r = i / P, pc = i % P;
    const int64_t ch = ch_base + pc * EPP;
    const bool ok = ch < channels;
    bwd_cp_async(dst + (uint32_t)(r * 32 * (int)sizeof(TIO) + pc * 16),
                 ok ? (const void*)(src + (tok0 + r) * channels + ch) : (const void*)src, ok ? 16 : 0);
  }
}

// Stage `nbytes` (a multiple of 16) contiguous bytes
__device__ __forceinline__ void bwd_stage_contig(uint32_t dst, const void* src, int nbytes, int lane) {
  for (int i = lane * 16; i < nbytes; i += 32 * 16) bwd_cp_async(dst + i, static_cast<const char*>(src) + i, 16);
}

// Bytes of one warp's staged tile in the aggregate kernel: Delta and dy rows,
// then the C rows
template <typename TIO, int NS>
__host__ __device__ constexpr int bwd_agg_stage_bytes(int T) {
  return (2 * 32 + NS) * T * (int)sizeof(TIO);
}

// the B (or C) row of a token from shared memory as NS floats
template <typename TIO, int NS>
__device__ __forceinline__ void load_row_smem(const TIO* row, float (&v)[NS]) {
  if constexpr (sizeof(TIO) == 2 && NS % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NS / 8; ++i) {
      const uint4 w = reinterpret_cast<const uint4*>(row)[i];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
        v[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
      }
    }
  } else if constexpr (sizeof(TIO) == 4 && NS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NS / 4; ++i) {
      const float4 w = reinterpret_cast<const float4*>(row)[i];
      v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int n = 0; n < NS; ++n) v[n] = to_f32(row[n]);
  }
}

// the B (or C) row of a token as NS floats: vector loads of the raw row
template <typename TIO, int NS>
__device__ __forceinline__ void load_row(const TIO* row, float (&v)[NS], bool vec) {
  if (!vec) {
#pragma unroll
    for (int n = 0; n < NS; ++n) v[n] = to_f32(row[n]);
    return;
  }
  if constexpr (sizeof(TIO) == 2) {
    if constexpr (NS % 8 == 0) {
#pragma unroll
      for (int i = 0; i < NS / 8; ++i) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(row) + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
          v[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int n = 0; n < NS; ++n) v[n] = to_f32(row[n]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < NS / 4; ++i) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(row) + i);
      v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
    }
  }
}

// Sum over the 32 lanes of v[0..31]; lane i returns the sum of v[i]
// (butterfly reduce-scatter: at each step a lane keeps the half of its
// values whose index has the lane's bit, and receives the partner's copy).
// The state scratch is written once and read once per half tile: its
// stores ask L2 to keep the lines (evict-last policy), and once a slot has
// been read its lines are discarded from L2, so that dead states are never
// written back to DRAM.
__device__ __forceinline__ uint64_t l2_keep_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_keep(float* p, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void l2_discard128(const void* p) {  // p: 128-byte aligned
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

constexpr int kBwdWarps = 4;  // warps per CTA of the backward kernel
// resident CTAs per SM of the reverse kernel: the per-warp state scratch of
// all resident warps should stay in L2
#ifndef MAMBA_BWD_CTAS_PER_SM
#define MAMBA_BWD_CTAS_PER_SM 2
#endif
constexpr int kBwdCtasPerSm = MAMBA_BWD_CTAS_PER_SM;

// q_n = exp(Delta A_n) - 1 for all states of one lane and token.  STRUCT
// (A[d,n] = (n+1) A[d,0] on every lane of the warp): one accurate expm1 and
// the decay chain of the forward kernel; otherwise one expm1 per state.
template <int NS, bool STRUCT>
__device__ __forceinline__ void decays(float dt, const float (&An)[NS], float (&q)[NS]) {
  if constexpr (STRUCT) {
    const float q0 = expm1_small(dt * An[0]);
    float2 e2[NS / 2];
    decay_chain<NS>(1.0f + q0, q0, e2);
#pragma unroll
    for (int k = 0; k < NS / 2; ++k) {
      q[2 * k] = e2[k].x;
      q[2 * k + 1] = e2[k].y;
    }
  } else {
#pragma unroll
    for (int n = 0; n < NS; ++n) q[n] = expm1_small(dt * An[n]);
  }
}

// psi(z) = (z e^z - (e^z - 1)) / z^2 = d/dA [(e^{Delta A} - 1)/A] / Delta^2,
// given q = e^z - 1.  The closed form cancels for small |z| (relative error
// about 2 eps / |z|), so |z| <= 1/4 takes the series
// sum_k (k+1) z^k / (k+2)! through z^6 (truncation below 3e-9 relative).
__device__ __forceinline__ float psi_f(float z, float q) {
  float s = fmaf(z, 1.0f / 5760.0f, 1.0f / 840.0f);
  s = fmaf(z, s, 1.0f / 144.0f);
  s = fmaf(z, s, 1.0f / 30.0f);
  s = fmaf(z, s, 1.0f / 8.0f);
  s = fmaf(z, s, 1.0f / 3.0f);
  s = fmaf(z, s, 0.5f);
  const float closed = (fmaf(z, q, z) - q) / (z * z);
  return fabsf(z) <= 0.25f ? s : closed;
}

// A work item's channel group has structured A (every lane, exact fp32 test)
template <int NS>
__device__ __forceinline__ bool group_structured(const float (&An)[NS]) {
  bool ok = An[0] < 0.0f;
#pragma unroll
  for (int n = 1; n < NS; ++n) ok &= (An[n] == (float)(n + 1) * An[0]);
  return __all_sync(0xffffffffu, ok);
}

// Outgoing adjoint of super-chunk j >= 1 from a zero incoming adjoint, M_j
// (after its first token, multiplied by that token's exp(Delta A)), and its
// sum of Delta: the reverse counterpart of the forward aggregates.  Only C,
// dy and Delta enter (no state).
template <typename TIO, int NS, bool STRUCT, bool STAGED>
__device__ __forceinline__ void bwd_aggregate_item(const BwdArgs<TIO>& a, int j, int64_t stream, int64_t b,
                                                   int64_t d, bool active, int lane, const float (&An)[NS],
                                                   TIO* stg) {
  const int64_t streams = a.batch * a.groups_d;
  const int T = a.tile;
  const int64_t t_lo = (int64_t)j * a.super_tiles * T;
  const int64_t t_hi = (j == a.supers - 1) ? a.len : (int64_t)(j + 1) * a.super_tiles * T;
  float mu[NS];
#pragma unroll
  for (int n = 0; n < NS; ++n) mu[n] = 0.0f;
  float sd = 0.0f;
  // tiles in reverse (t_lo is a tile boundary; the last tile may be short)
  for (int64_t tt0 = t_lo + ((t_hi - 1 - t_lo) / T) * T; tt0 >= t_lo; tt0 -= T) {
    const int rows = (int)(t_hi - tt0 < (int64_t)T ? t_hi - tt0 : (int64_t)T);
    const TIO* sdl = stg;  // staged rows: Delta, dy [T][32], then C [T][NS]
    const TIO* sdy = stg + T * 32;
    const TIO* sC = stg + 2 * T * 32;
    if constexpr (STAGED) {
      __syncwarp();
      constexpr int RB = 32 * (int)sizeof(TIO);
      const uint32_t s0 = smem_addr(stg);
      const int64_t tok0 = b * a.len + tt0;
      bwd_stage_rows<TIO>(s0, a.delta, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + T * RB, a.dy, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_contig(s0 + 2 * T * RB, a.C + tok0 * NS, rows * NS * (int)sizeof(TIO), lane);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncwarp();
    }
    for (int k = rows - 1; k >= 0; --k) {
      const int64_t tok = b * a.len + tt0 + k;
      float dt, gy, cv[NS], q[NS];
      if constexpr (STAGED) {
        dt = to_f32(sdl[k * 32 + lane]);
        gy = to_f32(sdy[k * 32 + lane]);
        load_row_smem<TIO, NS>(sC + k * NS, cv);
      } else {
        dt = active ? to_f32(a.delta[tok * a.channels + d]) : 0.0f;
        gy = active ? to_f32(a.dy[tok * a.channels + d]) : 0.0f;
        load_row<TIO, NS>(a.C + tok * NS, cv, a.vec_rows);
      }
      decays<NS, STRUCT>(dt, An, q);
      sd += dt;
#pragma unroll
      for (int n = 0; n < NS; ++n) mu[n] = (1.0f + q[n]) * fmaf(cv[n], gy, mu[n]);
    }
  }
  const size_t base = ((size_t)j * streams + stream) * 32 + lane;
  a.agg_sd[base] = sd;
#pragma unroll
  for (int n = 0; n < NS; ++n) a.agg_mu[base * NS + n] = mu[n];
}

template <typename TIO, int NS>
__global__ void __launch_bounds__(kBwdWarps * 32)
scan_backward_aggregate_kernel(const BwdArgs<TIO> a) {
  extern __shared__ __align__(16) unsigned char bwd_agg_smem[];
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TIO* stg = reinterpret_cast<TIO*>(bwd_agg_smem + warp * bwd_agg_stage_bytes<TIO, NS>(a.tile));
  const int64_t streams = a.batch * a.groups_d;
  const int64_t item = (int64_t)blockIdx.x * kBwdWarps + warp;  // (j - 1) * streams + stream
  if (item >= (int64_t)(a.supers - 1) * streams) return;
  const int j = 1 + (int)(item / streams);
  const int64_t stream = item - (int64_t)(j - 1) * streams;
  const int64_t b = stream / a.groups_d;
  const int64_t d = (stream - b * a.groups_d) * 32 + lane;
  const bool active = d < a.channels;
  float An[NS];
#pragma unroll
  for (int n = 0; n < NS; ++n) An[n] = active ? __ldg(a.A + d * NS + n) : -(float)(n + 1);
  const bool st = group_structured<NS>(An);
  if (a.staged) {
    if (st) bwd_aggregate_item<TIO, NS, true, true>(a, j, stream, b, d, active, lane, An, stg);
    else bwd_aggregate_item<TIO, NS, false, true>(a, j, stream, b, d, active, lane, An, stg);
  } else {
    if (st) bwd_aggregate_item<TIO, NS, true, false>(a, j, stream, b, d, active, lane, An, stg);
    else bwd_aggregate_item<TIO, NS, false, false>(a, j, stream, b, d, active, lane, An, stg);
  }
}

// One work item: super-chunk j of one stream, tiles in reverse.  STAGED:
// the tile's inputs are copied to `stg` (this warp's shared memory) first.
template <typename TIO, int NS, bool STRUCT, bool STAGED>
__device__ __forceinline__ void bwd_item(const BwdArgs<TIO>& a, int j, int64_t stream, int64_t b, int64_t d,
                                         bool active, int lane, const float (&An)[NS], float* S, TIO* stg) {
  const int64_t streams = a.batch * a.groups_d;
  const int T = a.tile;
  const int64_t ntiles = (a.len + T - 1) / T;
  const uint64_t keep = l2_keep_policy();  // for the state scratch
  // adjoints lam and the dA sums in pairs of states (n, n+1), so that the
  // reverse step runs as packed FFMA2; LAM(n) / DA(n) / IA(n) name one state
  float2 lam2[NS / 2], dA2[NS / 2], iA2[NS / 2], An2[NS / 2];
  auto LAM = [&](int n) -> float& { return (n & 1) ? lam2[n >> 1].y : lam2[n >> 1].x; };
  auto DA = [&](int n) -> float& { return (n & 1) ? dA2[n >> 1].y : dA2[n >> 1].x; };
  auto IA = [&](int n) -> float { return (n & 1) ? iA2[n >> 1].y : iA2[n >> 1].x; };
#pragma unroll
  for (int p = 0; p < NS / 2; ++p) {
    An2[p] = make_float2(An[2 * p], An[2 * p + 1]);
    iA2[p] = make_float2(1.0f / An[2 * p], 1.0f / An[2 * p + 1]);
    dA2[p] = make_float2(0.0f, 0.0f);
  }
#pragma unroll
  for (int n = 0; n < NS; ++n) LAM(n) = (active && a.dh_final) ? a.dh_final[(b * a.channels + d) * NS + n] : 0.0f;
  // the adjoint entering super-chunk j from the later ones:
  //   mu <- M_k + exp(A sumDelta_k) mu,  k = S-1 .. j+1,  mu_S = d h_final
  for (int k = a.supers - 1; k > j; --k) {
    const size_t base = ((size_t)k * streams + stream) * 32 + lane;
    const float sdk = a.agg_sd[base];
#pragma unroll
    for (int n = 0; n < NS; ++n) LAM(n) = fmaf(expf(An[n] * sdk), LAM(n), a.agg_mu[base * NS + n]);
  }
  const float Dd = (active && a.D) ? __ldg(a.D + d) : 0.0f;
  float dD = 0.0f;

  const int64_t tile_lo = (int64_t)j * a.super_tiles;
  const int64_t tile_hi = (j == a.supers - 1) ? ntiles : tile_lo + a.super_tiles;
  for (int64_t tile = tile_hi - 1; tile >= tile_lo; --tile) {
    const int64_t t0 = tile * T;
    const int rows = (int)(a.len - t0 < (int64_t)T ? a.len - t0 : (int64_t)T);
    const float* ck = a.ckpt + ((b * ntiles + tile) * a.channels + (active ? d : 0)) * NS;
    const TIO* su = stg;                 // staged rows: u, Delta, dy [T][32], then B, C [T][NS]
    const TIO* sdl = stg + T * 32;
    const TIO* sdy = stg + 2 * T * 32;
    const TIO* sB = stg + 3 * T * 32;
    const TIO* sC = sB + T * NS;
    if constexpr (STAGED) {
      __syncwarp();  // every lane is done with the previous tile's rows
      constexpr int RB = 32 * (int)sizeof(TIO);  // bytes per staged row
      const uint32_t s0 = smem_addr(stg);
      const int64_t tok0 = b * a.len + t0;
      bwd_stage_rows<TIO>(s0, a.u, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + T * RB, a.delta, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + 2 * T * RB, a.dy, tok0, rows, d - lane, a.channels, lane);
      const uint32_t sbB = s0 + 3 * T * RB, sbC = sbB + T * NS * (int)sizeof(TIO);
      bwd_stage_contig(sbB, a.B + tok0 * NS, rows * NS * (int)sizeof(TIO), lane);
      bwd_stage_contig(sbC, a.C + tok0 * NS, rows * NS * (int)sizeof(TIO), lane);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncwarp();
    }
    auto get_x = [&](int k, int64_t tok) -> float {
      if constexpr (STAGED) return to_f32(su[k * 32 + lane]);
      else return active ? to_f32(a.u[tok * a.channels + d]) : 0.0f;
    };
    auto get_dt = [&](int k, int64_t tok) -> float {
      if constexpr (STAGED) return to_f32(sdl[k * 32 + lane]);
      else return active ? to_f32(a.delta[tok * a.channels + d]) : 0.0f;
    };
    auto get_dy = [&](int k, int64_t tok) -> float {
      if constexpr (STAGED) return to_f32(sdy[k * 32 + lane]);
      else return active ? to_f32(a.dy[tok * a.channels + d]) : 0.0f;
    };
    auto get_B = [&](int k, int64_t tok, float (&v)[NS]) {
      if constexpr (STAGED) load_row_smem<TIO, NS>(sB + k * NS, v);
      else load_row<TIO, NS>(a.B + tok * NS, v, a.vec_rows);
    };
    auto get_C = [&](int k, int64_t tok, float (&v)[NS]) {
      if constexpr (STAGED) load_row_smem<TIO, NS>(sC + k * NS, v);
      else load_row<TIO, NS>(a.C + tok * NS, v, a.vec_rows);
    };
    // The tile goes in two halves, the later one first, so that the scratch
    // holds half a tile of states (and stays in L2): for each half, a
    // forward pass from the checkpoint through the half's end keeps
    // S[0] = h before the half's first token and S[1 + i] = h after its
    // token i; the reverse steps then read h_{t-1} from S one token ahead.
    const int H = T / 2;
    for (int half = 1; half >= 0; --half) {
    const int start = half * H;
    if (start >= rows) continue;
    const int end = (start + H < rows) ? start + H : rows;
    auto put = [&](int slot, const float (&v)[NS]) {
#pragma unroll
      for (int n = 0; n < NS; n += 4)
        st_keep(S + (size_t)slot * 32 * NS + n, make_float4(v[n], v[n + 1], v[n + 2], v[n + 3]), keep);
    };
    float h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) h[n] = active ? ck[n] : 0.0f;
    if (start == 0) put(0, h);
    for (int k = 0; k < end; ++k) {
      const int64_t tok = b * a.len + t0 + k;
      const float x = get_x(k, tok);
      const float dt = get_dt(k, tok);
      float bv[NS], q[NS];
      get_B(k, tok, bv);
      decays<NS, STRUCT>(dt, An, q);
#pragma unroll
      for (int n = 0; n < NS; ++n) h[n] = fmaf(1.0f + q[n], h[n], q[n] * IA(n) * bv[n] * x);
      if (k == start - 1) put(0, h);
      if (k >= start && k < end - 1) put(k - start + 1, h);  // (h after the half's last token: kept in h)
    }
    // reverse over the half; h holds h_t, hp is read back as h_{t-1}, one
    // token ahead of its use (hn)
    auto read_prev = [&](int k, float (&v)[NS]) {  // h_{t0+k-1}
#pragma unroll
      for (int n = 0; n < NS; n += 4) {
        const float4 w = *reinterpret_cast<const float4*>(S + (size_t)(k - start) * 32 * NS + n);
        v[n] = w.x; v[n + 1] = w.y; v[n + 2] = w.z; v[n + 3] = w.w;
      }
    };
    float hn[NS];
    read_prev(end - 1, hn);
    for (int k = end - 1; k >= start; --k) {
      const int64_t tok = b * a.len + t0 + k;
      float hp[NS];
#pragma unroll
      for (int n = 0; n < NS; ++n) hp[n] = hn[n];
      if (k > start) read_prev(k - 1, hn);
      const float x = get_x(k, tok);
      const float dt = get_dt(k, tok);
      const float gy = get_dy(k, tok);
      float du = Dd * gy, ddt = 0.0f;
      dD = fmaf(gy, x, dD);
      float bv[NS], cv[NS];
      get_B(k, tok, bv);
      get_C(k, tok, cv);
      // structured A: q_n from the decay chain, and d_n = q_n - z_n exactly
      // from d_n = e^{z_0} d_{n-1} + n z_0 q_0 + d_0 (every term of one sign,
      // so nothing cancels); the B x part of dA_n is then
      // B x Delta^2 psi(z_n) = B x (z_n q_n - d_n) / A_n^2
      float red[32];
      if constexpr (STRUCT) {
        // q_n from the decay chain, and nd_n = -(q_n - z_n) exactly from
        // d_n = e^{z_0} d_{n-1} + n z_0 q_0 + d_0 (every term of one sign, so
        // nothing cancels); the B x part of dA_n is then
        // B x Delta^2 psi(z_n) = B x (z_n q_n - d_n) / A_n^2.  Pairs of
        // states go through packed FFMA2.
        float q0, d0;
        expm1_parts(dt * An[0], q0, d0);
        float2 e2[NS / 2];
        decay_chain<NS>(1.0f + q0, q0, e2);
        const float r0 = 1.0f + q0, zq0 = dt * An[0] * q0;
        float nd[NS];
        nd[0] = -d0;
#pragma unroll
        for (int n = 1; n < NS; ++n) nd[n] = fmaf(r0, nd[n - 1], fmaf(-(float)n, zq0, -d0));
        const float2 x2 = make_float2(x, x), gy2 = make_float2(gy, gy), dt2 = make_float2(dt, dt);
        const float2 one2 = make_float2(1.0f, 1.0f);
        float2 du2 = make_float2(0.0f, 0.0f), ddt2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int pp = 0; pp < NS / 2; ++pp) {
          const int n = 2 * pp;
          const float2 q2 = e2[pp];
          const float2 r2 = __fadd2_rn(q2, one2);
          const float2 b2 = make_float2(bv[n], bv[n + 1]);
          const float2 c2 = make_float2(cv[n], cv[n + 1]);
          const float2 hp2 = make_float2(hp[n], hp[n + 1]);
          const float2 bx2 = __fmul2_rn(b2, x2);
          const float2 qa2 = __fmul2_rn(q2, iA2[pp]);
          const float2 rc = __fmul2_rn(gy2, make_float2(h[n], h[n + 1]));  // dC_{t,n} part: dy_t h_t
          red[NS + n] = rc.x;
          red[NS + n + 1] = rc.y;
          const float2 L = __ffma2_rn(c2, gy2, lam2[pp]);
          du2 = __ffma2_rn(L, __fmul2_rn(qa2, b2), du2);
          ddt2 = __ffma2_rn(__fmul2_rn(L, r2), __ffma2_rn(An2[pp], hp2, bx2), ddt2);
          // d h_t / d A_n = Delta r h_{t-1} + B x Delta^2 psi(Delta A_n)
          const float2 z2 = __fmul2_rn(dt2, An2[pp]);
          const float2 bpsi2 = __fmul2_rn(bx2, __fmul2_rn(__ffma2_rn(z2, q2, make_float2(nd[n], nd[n + 1])),
                                                          __fmul2_rn(iA2[pp], iA2[pp])));
          dA2[pp] = __ffma2_rn(L, __ffma2_rn(__fmul2_rn(dt2, r2), hp2, bpsi2), dA2[pp]);
          const float2 rb = __fmul2_rn(__fmul2_rn(L, x2), qa2);  // dB_{t,n} part
          red[n] = rb.x;
          red[n + 1] = rb.y;
          lam2[pp] = __fmul2_rn(L, r2);
          h[n] = hp[n];
          h[n + 1] = hp[n + 1];
        }
        du += du2.x + du2.y;
        ddt = ddt2.x + ddt2.y;
      } else {
        float q[NS];
        decays<NS, STRUCT>(dt, An, q);
#pragma unroll
        for (int n = 0; n < NS; ++n) {
          const float r = 1.0f + q[n];
          const float bx = bv[n] * x;
          const float qa = q[n] * IA(n);
          red[NS + n] = gy * h[n];                      // dC_{t,n} part: dy_t h_t
          LAM(n) = fmaf(cv[n], gy, LAM(n));
          du = fmaf(LAM(n), qa * bv[n], du);
          ddt = fmaf(LAM(n) * r, fmaf(An[n], hp[n], bx), ddt);
          // d h_t / d A_n = Delta r h_{t-1} + B x Delta^2 psi(Delta A_n)
          const float bpsi = bx * (dt * dt) * psi_f(dt * An[n], q[n]);
          DA(n) = fmaf(LAM(n), fmaf(dt * r, hp[n], bpsi), DA(n));
          red[n] = LAM(n) * x * qa;                     // dB_{t,n} part
          LAM(n) *= r;
          h[n] = hp[n];
        }
      }
#pragma unroll
      for (int n = 2 * NS; n < 32; ++n) red[n] = 0.0f;
      if (active) {
        a.du[tok * a.channels + d] = from_f32<TIO>(du);
        a.ddelta[tok * a.channels + d] = from_f32<TIO>(ddt);
      }
      const float s = reduce_scatter32(red, lane);
      if (lane < NS) atomicAdd(a.dB + tok * NS + lane, s);
      else if (lane < 2 * NS) atomicAdd(a.dC + tok * NS + (lane - NS), s);
      // slot k - start (h_{t-1} of this token) has been read by every lane:
      // drop its NS lines of 128 bytes from L2 without a write-back
      __syncwarp();
      if (lane < NS) l2_discard128(S - (size_t)lane * NS + (size_t)(k - start) * 32 * NS + (size_t)lane * 32);
    }
    __syncwarp();  // every discard before the next half's stores into the same lines
    }  // half
  }
  if (active) {
#pragma unroll
    for (int n = 0; n < NS; ++n) atomicAdd(a.dA + d * NS + n, DA(n));
    if (a.dD) atomicAdd(a.dD + d, dD);
    if (a.dh0 && j == 0) {
#pragma unroll
      for (int n = 0; n < NS; ++n) a.dh0[(b * a.channels + d) * NS + n] = LAM(n);
    }
  }
}

// at least three CTAs per SM: the occupancy is worth a few spilled registers
template <typename TIO, int NS>
__global__ void __launch_bounds__(kBwdWarps * 32, kBwdCtasPerSm)
scan_backward_kernel(const BwdArgs<TIO> a) {
  static_assert(2 * NS <= 32, "dB and dC of a token are reduced in one 32-lane pass");
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  griddep_wait();  // the aggregates and checkpoints come from the previous kernels of the stream
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TIO* stg = reinterpret_cast<TIO*>(bwd_smem + warp * bwd_stage_bytes<TIO, NS>(a.tile));
  const int64_t wid = (int64_t)blockIdx.x * kBwdWarps + warp;
  const int64_t nwarps = (int64_t)gridDim.x * kBwdWarps;
  const int64_t streams = a.batch * a.groups_d;
  float* S = a.scratch + (size_t)wid * (size_t)(a.tile / 2 + 1) * 32 * NS + (size_t)lane * NS;  // + k * 32 * NS
  // work item = (super-chunk j, stream), the later super-chunks first
  for (int64_t item = wid; item < (int64_t)a.supers * streams; item += nwarps) {
    const int j = a.supers - 1 - (int)(item / streams);
    const int64_t stream = item - (int64_t)(a.supers - 1 - j) * streams;
    const int64_t b = stream / a.groups_d;
    const int64_t d = (stream - b * a.groups_d) * 32 + lane;
    const bool active = d < a.channels;
    float An[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) An[n] = active ? __ldg(a.A + d * NS + n) : -(float)(n + 1);
    const bool st = group_structured<NS>(An);
    if (a.staged) {
      if (st) bwd_item<TIO, NS, true, true>(a, j, stream, b, d, active, lane, An, S, stg);
      else bwd_item<TIO, NS, false, true>(a, j, stream, b, d, active, lane, An, S, stg);
    } else {
      if (st) bwd_item<TIO, NS, true, false>(a, j, stream, b, d, active, lane, An, S, stg);
      else bwd_item<TIO, NS, false, false>(a, j, stream, b, d, active, lane, An, S, stg);
    }
  }
}

}  // namespace mamba
