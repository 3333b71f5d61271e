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
// warps, so it stays in L2), then walks the half in reverse.  Every
// per-state quantity is a pair of states in one 64-bit register pair, so
// that both passes run as packed FFMA2.  dB and dC of a token are sums over
// the warp's 32 channels: each lane writes its 2N parts as one column of a
// 32 x 32 transpose area in shared memory, lane j < 2N adds row j, and adds
// it to global memory with one atomic.  bf16 B and C are widened to
// fp32 once (a small kernel ahead of the forward pass).  When rows are
// 16-byte aligned, the warp first copies the tile's u, Delta and dy rows and
// its fp32 B, C rows into its shared memory (one round of 16-byte cp.async
// copies), so both passes over the tile read shared memory instead of
// waiting on a global load per token.
#pragma once

#include "common.cuh"
#include "scan.cuh"  // expm1_small

namespace mamba {

template <typename TIO>
struct BwdArgs {
  const TIO* u;
  const TIO* delta;
  const float* A;
  const float* Bf;         // [batch][len][N] B as fp32 (the input itself, or a widened copy of bf16 B)
  const float* Cf;         // [batch][len][N] C as fp32
  const float* D;          // nullable
  const TIO* dy;
  const float* dh_final;   // nullable
  const float* ckpt;       // [batch][ntiles][channels][N]
  float* scratch;          // [warps of the grid][T/2 + 1][32][N]
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
  int vec_rows;            // fp32 B and C rows may be read with 16-byte vector loads
  int supers;              // S: the sequence is cut into S super-chunks of super_tiles tiles
  int super_tiles;
  float* agg_mu;           // [S][streams][32][N] outgoing adjoint of super-chunk j from zero
  float* agg_sd;           // [S][streams][32] sum of Delta over super-chunk j
  int staged;              // tiles are staged in shared memory (rows 16-byte aligned)
};

// bf16 B and C rows widened to fp32 once, so that the reverse kernels read
// whole fp32 rows (the 16-byte pieces of both arrays when aligned, else one
// element per step)
__global__ void bwd_widen_kernel(const __nv_bfloat16* __restrict__ B, const __nv_bfloat16* __restrict__ C,
                                 float* __restrict__ Bf, float* __restrict__ Cf, int64_t n, int vec) {
  griddep_wait();  // B and C may come from the previous kernel of the stream
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (vec) {  // both arrays 16-byte aligned and n a multiple of 8
    for (int64_t i = i0; i < n / 8; i += stride) {
      const uint4 wb = __ldg(reinterpret_cast<const uint4*>(B) + i);
      const uint4 wc = __ldg(reinterpret_cast<const uint4*>(C) + i);
      auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
      auto hi = [](uint32_t w) { return __uint_as_float(w & 0xffff0000u); };
      float4* ob = reinterpret_cast<float4*>(Bf) + 2 * i;
      float4* oc = reinterpret_cast<float4*>(Cf) + 2 * i;
      ob[0] = make_float4(lo(wb.x), hi(wb.x), lo(wb.y), hi(wb.y));
      ob[1] = make_float4(lo(wb.z), hi(wb.z), lo(wb.w), hi(wb.w));
      oc[0] = make_float4(lo(wc.x), hi(wc.x), lo(wc.y), hi(wc.y));
      oc[1] = make_float4(lo(wc.z), hi(wc.z), lo(wc.w), hi(wc.w));
    }
  } else {
    for (int64_t i = i0; i < n; i += stride) {
      Bf[i] = __bfloat162float(B[i]);
      Cf[i] = __bfloat162float(C[i]);
    }
  }
}

// Per warp of the reverse kernels: a 32 x 32 fp32 transpose area for the
// dB / dC sums of a token, then (staged tiles) the tile's rows.
constexpr int kBwdRedBytes = 32 * 32 * (int)sizeof(float);

// Bytes of one warp's staged tile: u, Delta and dy rows of 32 channels, then
// the fp32 B and C rows, for T tokens.
template <typename TIO, int NS>
__host__ __device__ constexpr int bwd_stage_bytes(int T) {
  return 3 * 32 * T * (int)sizeof(TIO) + 2 * NS * T * (int)sizeof(float);
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
// then the fp32 C rows
template <typename TIO, int NS>
__host__ __device__ constexpr int bwd_agg_stage_bytes(int T) {
  return 2 * 32 * T * (int)sizeof(TIO) + NS * T * (int)sizeof(float);
}

// An fp32 B (or C) row of a token as NS/2 pairs: from shared memory (16-byte
// aligned), or from global memory with vector loads when `vec`
template <int NS>
__device__ __forceinline__ void row_pairs_smem(const float* row, float2 (&v)[NS / 2]) {
  if constexpr (NS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NS / 4; ++i) {
      const float4 w = reinterpret_cast<const float4*>(row)[i];
      v[2 * i] = make_float2(w.x, w.y);
      v[2 * i + 1] = make_float2(w.z, w.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) v[i] = make_float2(row[2 * i], row[2 * i + 1]);
  }
}
template <int NS>
__device__ __forceinline__ void row_pairs_global(const float* row, float2 (&v)[NS / 2], bool vec) {
  if constexpr (NS % 4 == 0) {
    if (vec) {
#pragma unroll
      for (int i = 0; i < NS / 4; ++i) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(row) + i);
        v[2 * i] = make_float2(w.x, w.y);
        v[2 * i + 1] = make_float2(w.z, w.w);
      }
      return;
    }
  }
#pragma unroll
  for (int i = 0; i < NS / 2; ++i) v[i] = make_float2(__ldg(row + 2 * i), __ldg(row + 2 * i + 1));
}

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

// The dB / dC sums of one token over the warp's 32 channels go through a
// transpose in shared memory: value c of lane i is stored at c * 32 + i (a
// row per value; the 32 lanes' stores of one value fill the 32 banks), and
// lane j < 2N adds row j with eight 16-byte loads.  Lane j takes the row's
// pieces in the order j, j+1, ... (mod 8), so that the eight lanes of a
// quarter-warp read eight distinct 4-bank groups at each load.
__device__ __forceinline__ float red_row_sum(const float* red, int row) {
  const float4* r = reinterpret_cast<const float4*>(red + row * 32);
  float2 s0 = make_float2(0.0f, 0.0f), s1 = s0;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float4 v = r[(m + row) & 7];
    s0 = __fadd2_rn(s0, make_float2(v.x, v.y));
    s1 = __fadd2_rn(s1, make_float2(v.z, v.w));
  }
  s0 = __fadd2_rn(s0, s1);
  return s0.x + s0.y;
}

constexpr int kBwdWarps = 4;  // warps per CTA of the backward kernel
// resident CTAs per SM of the reverse kernel: the per-warp state scratch of
// all resident warps should stay in L2
#ifndef MAMBA_BWD_CTAS_PER_SM
#define MAMBA_BWD_CTAS_PER_SM 2
#endif
constexpr int kBwdCtasPerSm = MAMBA_BWD_CTAS_PER_SM;

// q_n = exp(Delta A_n) - 1 for all states of one lane and token, as pairs
// (q_{2k}, q_{2k+1}).  STRUCT (A[d,n] = (n+1) A[d,0] on every lane of the
// warp): one accurate expm1 and the decay chain of the forward kernel;
// otherwise one expm1 per state.
template <int NS, bool STRUCT>
__device__ __forceinline__ void decays(float dt, const float (&An)[NS], float2 (&q)[NS / 2]) {
  if constexpr (STRUCT) {
    const float q0 = expm1_small(dt * An[0]);
    decay_chain<NS>(1.0f + q0, q0, q);
  } else {
#pragma unroll
    for (int k = 0; k < NS / 2; ++k) q[k] = make_float2(expm1_small(dt * An[2 * k]), expm1_small(dt * An[2 * k + 1]));
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

// one state of an array of pairs (n is a compile-time index after unrolling)
__device__ __forceinline__ float& st_of(float2* v, int n) { return (n & 1) ? v[n >> 1].y : v[n >> 1].x; }

// Outgoing adjoint of super-chunk j >= 1 from a zero incoming adjoint, M_j
// (after its first token, multiplied by that token's exp(Delta A)), and its
// sum of Delta: the reverse counterpart of the forward aggregates.  Only C,
// dy and Delta enter (no state).
template <typename TIO, int NS, bool STRUCT, bool STAGED>
__device__ __forceinline__ void bwd_aggregate_item(const BwdArgs<TIO>& a, int j, int64_t stream, int64_t b,
                                                   int64_t d, bool active, int lane, const float (&An)[NS],
                                                   unsigned char* stg) {
  constexpr int P = NS / 2;
  const int64_t streams = a.batch * a.groups_d;
  const int T = a.tile;
  const int64_t t_lo = (int64_t)j * a.super_tiles * T;
  const int64_t t_hi = (j == a.supers - 1) ? a.len : (int64_t)(j + 1) * a.super_tiles * T;
  float2 mu[P];
#pragma unroll
  for (int p = 0; p < P; ++p) mu[p] = make_float2(0.0f, 0.0f);
  float sd = 0.0f;
  const TIO* sdl = reinterpret_cast<const TIO*>(stg);  // staged rows: Delta, dy [T][32], then fp32 C [T][NS]
  const TIO* sdy = sdl + T * 32;
  const float* sC = reinterpret_cast<const float*>(stg + 2 * T * 32 * (int)sizeof(TIO));
  // tiles in reverse (t_lo is a tile boundary; the last tile may be short)
  for (int64_t tt0 = t_lo + ((t_hi - 1 - t_lo) / T) * T; tt0 >= t_lo; tt0 -= T) {
    const int rows = (int)(t_hi - tt0 < (int64_t)T ? t_hi - tt0 : (int64_t)T);
    if constexpr (STAGED) {
      __syncwarp();
      constexpr int RB = 32 * (int)sizeof(TIO);
      const uint32_t s0 = smem_addr(stg);
      const int64_t tok0 = b * a.len + tt0;
      bwd_stage_rows<TIO>(s0, a.delta, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + T * RB, a.dy, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_contig(s0 + 2 * T * RB, a.Cf + tok0 * NS, rows * NS * (int)sizeof(float), lane);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncwarp();
    }
    for (int k = rows - 1; k >= 0; --k) {
      const int64_t tok = b * a.len + tt0 + k;
      float dt, gy;
      float2 cv[P], q[P];
      if constexpr (STAGED) {
        dt = to_f32(sdl[k * 32 + lane]);
        gy = to_f32(sdy[k * 32 + lane]);
        row_pairs_smem<NS>(sC + k * NS, cv);
      } else {
        dt = active ? to_f32(a.delta[tok * a.channels + d]) : 0.0f;
        gy = active ? to_f32(a.dy[tok * a.channels + d]) : 0.0f;
        row_pairs_global<NS>(a.Cf + tok * NS, cv, a.vec_rows);
      }
      decays<NS, STRUCT>(dt, An, q);
      sd += dt;
      const float2 gy2 = make_float2(gy, gy), one2 = make_float2(1.0f, 1.0f);
#pragma unroll
      for (int p = 0; p < P; ++p) mu[p] = __fmul2_rn(__fadd2_rn(q[p], one2), __ffma2_rn(cv[p], gy2, mu[p]));
    }
  }
  const size_t base = ((size_t)j * streams + stream) * 32 + lane;
  a.agg_sd[base] = sd;
#pragma unroll
  for (int n = 0; n < NS; ++n) a.agg_mu[base * NS + n] = st_of(mu, n);
}

template <typename TIO, int NS>
__global__ void __launch_bounds__(kBwdWarps * 32)
scan_backward_aggregate_kernel(const BwdArgs<TIO> a) {
  extern __shared__ __align__(16) unsigned char bwd_agg_smem[];
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* stg = bwd_agg_smem + warp * bwd_agg_stage_bytes<TIO, NS>(a.tile);
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

// One work item: super-chunk j of one stream, tiles in reverse.  `red` is
// this warp's transpose area; STAGED: the tile's inputs are copied to `stg`
// (this warp's shared memory) first.  Every per-state quantity is kept as
// N/2 pairs of states (n, n+1), so that the steps run as packed FFMA2.
template <typename TIO, int NS, bool STRUCT, bool STAGED>
__device__ __forceinline__ void bwd_item(const BwdArgs<TIO>& a, int j, int64_t stream, int64_t b, int64_t d,
                                         bool active, int lane, const float (&An)[NS], float* S, float* red,
                                         unsigned char* stg) {
  constexpr int P = NS / 2;
  const int64_t streams = a.batch * a.groups_d;
  const int T = a.tile;
  const int64_t ntiles = (a.len + T - 1) / T;
  const uint64_t keep = l2_keep_policy();  // for the state scratch
  // adjoints lam and the dA sums
  float2 lam2[P], dA2[P], iA2[P], An2[P];
#pragma unroll
  for (int p = 0; p < P; ++p) {
    An2[p] = make_float2(An[2 * p], An[2 * p + 1]);
    iA2[p] = make_float2(1.0f / An[2 * p], 1.0f / An[2 * p + 1]);
    dA2[p] = make_float2(0.0f, 0.0f);
  }
#pragma unroll
  for (int n = 0; n < NS; ++n)
    st_of(lam2, n) = (active && a.dh_final) ? a.dh_final[(b * a.channels + d) * NS + n] : 0.0f;
  // the adjoint entering super-chunk j from the later ones:
  //   mu <- M_k + exp(A sumDelta_k) mu,  k = S-1 .. j+1,  mu_S = d h_final
  for (int k = a.supers - 1; k > j; --k) {
    const size_t base = ((size_t)k * streams + stream) * 32 + lane;
    const float sdk = a.agg_sd[base];
#pragma unroll
    for (int n = 0; n < NS; ++n) st_of(lam2, n) = fmaf(expf(An[n] * sdk), st_of(lam2, n), a.agg_mu[base * NS + n]);
  }
  const float Dd = (active && a.D) ? __ldg(a.D + d) : 0.0f;
  float dD = 0.0f;
  const bool reducer = lane < 2 * NS;  // lane j < 2N sums row j (dB_j, or dC_{j-N})
  float* red_col = red + lane;         // this lane's column of the transpose area

  const TIO* su = reinterpret_cast<const TIO*>(stg);  // staged rows: u, Delta, dy [T][32], then fp32 B, C [T][NS]
  const TIO* sdl = su + T * 32;
  const TIO* sdy = su + 2 * T * 32;
  const float* sB = reinterpret_cast<const float*>(stg + 3 * T * 32 * (int)sizeof(TIO));
  const float* sC = sB + T * NS;
  const int64_t tile_lo = (int64_t)j * a.super_tiles;
  const int64_t tile_hi = (j == a.supers - 1) ? ntiles : tile_lo + a.super_tiles;
  for (int64_t tile = tile_hi - 1; tile >= tile_lo; --tile) {
    const int64_t t0 = tile * T;
    const int rows = (int)(a.len - t0 < (int64_t)T ? a.len - t0 : (int64_t)T);
    const float* ck = a.ckpt + ((b * ntiles + tile) * a.channels + (active ? d : 0)) * NS;
    if constexpr (STAGED) {
      __syncwarp();  // every lane is done with the previous tile's rows
      constexpr int RB = 32 * (int)sizeof(TIO);  // bytes per staged row
      const uint32_t s0 = smem_addr(stg);
      const int64_t tok0 = b * a.len + t0;
      bwd_stage_rows<TIO>(s0, a.u, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + T * RB, a.delta, tok0, rows, d - lane, a.channels, lane);
      bwd_stage_rows<TIO>(s0 + 2 * T * RB, a.dy, tok0, rows, d - lane, a.channels, lane);
      const uint32_t sbB = s0 + 3 * T * RB, sbC = sbB + T * NS * (int)sizeof(float);
      bwd_stage_contig(sbB, a.Bf + tok0 * NS, rows * NS * (int)sizeof(float), lane);
      bwd_stage_contig(sbC, a.Cf + tok0 * NS, rows * NS * (int)sizeof(float), lane);
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
    auto get_B = [&](int k, int64_t tok, float2 (&v)[P]) {
      if constexpr (STAGED) row_pairs_smem<NS>(sB + k * NS, v);
      else row_pairs_global<NS>(a.Bf + tok * NS, v, a.vec_rows);
    };
    auto get_C = [&](int k, int64_t tok, float2 (&v)[P]) {
      if constexpr (STAGED) row_pairs_smem<NS>(sC + k * NS, v);
      else row_pairs_global<NS>(a.Cf + tok * NS, v, a.vec_rows);
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
      auto put = [&](int slot, const float2 (&v)[P]) {
#pragma unroll
        for (int p = 0; p < P; p += 2)
          st_keep(S + (size_t)slot * 32 * NS + 2 * p, make_float4(v[p].x, v[p].y, v[p + 1].x, v[p + 1].y), keep);
      };
      float2 h2[P];
#pragma unroll
      for (int p = 0; p < P; p += 2) {
        const float4 w = active ? *reinterpret_cast<const float4*>(ck + 2 * p) : make_float4(0.f, 0.f, 0.f, 0.f);
        h2[p] = make_float2(w.x, w.y);
        h2[p + 1] = make_float2(w.z, w.w);
      }
      if (start == 0) put(0, h2);
      // forward: h <- h + q (h + B x / A), per pair of states three packed steps
      for (int k = 0; k < end; ++k) {
        const int64_t tok = b * a.len + t0 + k;
        const float x = get_x(k, tok);
        const float dt = get_dt(k, tok);
        float2 bv[P], q[P];
        get_B(k, tok, bv);
        decays<NS, STRUCT>(dt, An, q);
        const float2 x2 = make_float2(x, x);
#pragma unroll
        for (int p = 0; p < P; ++p)
          h2[p] = __ffma2_rn(q[p], __ffma2_rn(__fmul2_rn(bv[p], x2), iA2[p], h2[p]), h2[p]);
        if (k == start - 1) put(0, h2);
        if (k >= start && k < end - 1) put(k - start + 1, h2);  // (h after the half's last token: kept in h2)
      }
      // reverse over the half; h2 holds h_t, hn2 is read back as h_{t-1},
      // one token ahead of its use
      auto read_prev = [&](int k, float2 (&v)[P]) {  // h_{t0+k-1}
#pragma unroll
        for (int p = 0; p < P; p += 2) {
          const float4 w = *reinterpret_cast<const float4*>(S + (size_t)(k - start) * 32 * NS + 2 * p);
          v[p] = make_float2(w.x, w.y);
          v[p + 1] = make_float2(w.z, w.w);
        }
      };
      float2 hn2[P];
      read_prev(end - 1, hn2);
      for (int k = end - 1; k >= start; --k) {
        const int64_t tok = b * a.len + t0 + k;
        float2 hp2[P];
#pragma unroll
        for (int p = 0; p < P; ++p) hp2[p] = hn2[p];
        if (k > start) read_prev(k - 1, hn2);
        const float x = get_x(k, tok);
        const float dt = get_dt(k, tok);
        const float gy = get_dy(k, tok);
        float du = Dd * gy, ddt = 0.0f;
        dD = fmaf(gy, x, dD);
        float2 bv[P], cv[P];
        get_B(k, tok, bv);
        get_C(k, tok, cv);
        const float2 x2 = make_float2(x, x), gy2 = make_float2(gy, gy), dt2 = make_float2(dt, dt);
        const float2 one2 = make_float2(1.0f, 1.0f);
        // this token's parts of dB (L x q / A) and dC (dy h_t) of pair p into
        // this lane's column of the transpose area
        auto emit = [&](int p, float2 rb, float2 rc) {
          red_col[(2 * p) * 32] = rb.x;
          red_col[(2 * p + 1) * 32] = rb.y;
          red_col[(NS + 2 * p) * 32] = rc.x;
          red_col[(NS + 2 * p + 1) * 32] = rc.y;
        };
        if constexpr (STRUCT) {
          // q_n = Q_{n+1} from the decay chain, with Q_m = e^{m z_0} - 1, and
          // nd_n = -D_{n+1}, D_m = Q_m - m z_0, exactly from
          // D_{a+b} = D_a + D_b + Q_a Q_b (every term of one sign, so nothing
          // cancels): D_2..D_4 from D_1, then steps of four in pairs.  The
          // B x part of dA_n is then B x Delta^2 psi(z_n) = B x (z_n q_n - D_{n+1}) / A_n^2.
          float q0, d0;
          expm1_parts(dt * An[0], q0, d0);
          float2 e2[P];
          decay_chain<NS>(1.0f + q0, q0, e2);
          float2 nd2[P];
          {
            const float n1 = -d0;
            const float n2 = fmaf(-q0, q0, 2.0f * n1);
            const float n3 = fmaf(-e2[0].y, q0, n2 + n1);
            const float n4 = fmaf(-e2[1].x, q0, n3 + n1);
            nd2[0] = make_float2(n1, n2);
            nd2[1] = make_float2(n3, n4);
            const float2 n44 = make_float2(n4, n4), mq4 = make_float2(-e2[1].y, -e2[1].y);
#pragma unroll
            for (int p = 2; p < P; ++p) nd2[p] = __ffma2_rn(e2[p - 2], mq4, __fadd2_rn(nd2[p - 2], n44));
          }
          float2 du2 = make_float2(0.0f, 0.0f), ddt2 = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const float2 q2 = e2[p];
            const float2 r2 = __fadd2_rn(q2, one2);
            const float2 bx2 = __fmul2_rn(bv[p], x2);
            const float2 qa2 = __fmul2_rn(q2, iA2[p]);
            const float2 rc = __fmul2_rn(gy2, h2[p]);
            const float2 L = __ffma2_rn(cv[p], gy2, lam2[p]);
            const float2 U = __fmul2_rn(L, qa2);
            du2 = __ffma2_rn(U, bv[p], du2);
            const float2 rb = __fmul2_rn(U, x2);
            const float2 lr = __fmul2_rn(L, r2);
            ddt2 = __ffma2_rn(lr, __ffma2_rn(An2[p], hp2[p], bx2), ddt2);
            // d h_t / d A_n = Delta r h_{t-1} + B x Delta^2 psi(Delta A_n)
            const float2 z2 = __fmul2_rn(dt2, An2[p]);
            const float2 bpsi2 =
                __fmul2_rn(bx2, __fmul2_rn(__ffma2_rn(z2, q2, nd2[p]), __fmul2_rn(iA2[p], iA2[p])));
            dA2[p] = __ffma2_rn(L, __ffma2_rn(__fmul2_rn(dt2, r2), hp2[p], bpsi2), dA2[p]);
            lam2[p] = lr;
            h2[p] = hp2[p];
            emit(p, rb, rc);
          }
          du += du2.x + du2.y;
          ddt = ddt2.x + ddt2.y;
        } else {
          float2 q2[P];
          decays<NS, STRUCT>(dt, An, q2);
#pragma unroll
          for (int p = 0; p < P; ++p) {
            float2 rb, rc;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int n = 2 * p + e;
              const float q = e ? q2[p].y : q2[p].x;
              const float r = 1.0f + q;
              const float bn = e ? bv[p].y : bv[p].x;
              const float hp = e ? hp2[p].y : hp2[p].x;
              const float bx = bn * x;
              const float qa = q * (e ? iA2[p].y : iA2[p].x);
              const float L = fmaf(e ? cv[p].y : cv[p].x, gy, st_of(lam2, n));
              (e ? rc.y : rc.x) = gy * st_of(h2, n);  // dC_{t,n} part: dy_t h_t
              du = fmaf(L, qa * bn, du);
              ddt = fmaf(L * r, fmaf(An[n], hp, bx), ddt);
              // d h_t / d A_n = Delta r h_{t-1} + B x Delta^2 psi(Delta A_n)
              const float bpsi = bx * (dt * dt) * psi_f(dt * An[n], q);
              st_of(dA2, n) = fmaf(L, fmaf(dt * r, hp, bpsi), st_of(dA2, n));
              (e ? rb.y : rb.x) = L * x * qa;  // dB_{t,n} part
              st_of(lam2, n) = L * r;
            }
            h2[p] = hp2[p];
            emit(p, rb, rc);
          }
        }
        if (active) {
          a.du[tok * a.channels + d] = from_f32<TIO>(du);
          a.ddelta[tok * a.channels + d] = from_f32<TIO>(ddt);
        }
        __syncwarp();  // every row of the transpose area written
        if (reducer) {
          const float s = red_row_sum(red, lane);
          if (lane < NS) atomicAdd(a.dB + tok * NS + lane, s);
          else atomicAdd(a.dC + tok * NS + (lane - NS), s);
        }
        // slot k - start (h_{t-1} of this token) has been read by every lane,
        // and every row of the transpose area: drop the slot's NS lines
        // of 128 bytes from L2 without a write-back
        __syncwarp();
        if (lane < NS) l2_discard128(S - (size_t)lane * NS + (size_t)(k - start) * 32 * NS + (size_t)lane * 32);
      }
      __syncwarp();  // every discard before the next half's stores into the same lines
    }  // half
  }
  if (active) {
#pragma unroll
    for (int n = 0; n < NS; ++n) atomicAdd(a.dA + d * NS + n, st_of(dA2, n));
    if (a.dD) atomicAdd(a.dD + d, dD);
    if (a.dh0 && j == 0) {
#pragma unroll
      for (int n = 0; n < NS; ++n) a.dh0[(b * a.channels + d) * NS + n] = st_of(lam2, n);
    }
  }
}

// Per warp of the reverse kernel's shared memory: the transpose area, then
// (staged tiles) the tile's rows
template <typename TIO, int NS>
__host__ __device__ constexpr int bwd_warp_smem(int T, bool staged) {
  return kBwdRedBytes + (staged ? bwd_stage_bytes<TIO, NS>(T) : 0);
}

template <typename TIO, int NS>
__global__ void __launch_bounds__(kBwdWarps * 32, kBwdCtasPerSm)
scan_backward_kernel(const BwdArgs<TIO> a) {
  static_assert(2 * NS <= 32 && NS % 4 == 0, "dB and dC of a token are reduced in one 32-column transpose");
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  griddep_wait();  // the aggregates and checkpoints come from the previous kernels of the stream
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wsm = bwd_smem + warp * bwd_warp_smem<TIO, NS>(a.tile, a.staged != 0);
  float* red = reinterpret_cast<float*>(wsm);
  unsigned char* stg = wsm + kBwdRedBytes;
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
      if (st) bwd_item<TIO, NS, true, true>(a, j, stream, b, d, active, lane, An, S, red, stg);
      else bwd_item<TIO, NS, false, true>(a, j, stream, b, d, active, lane, An, S, red, stg);
    } else {
      if (st) bwd_item<TIO, NS, true, false>(a, j, stream, b, d, active, lane, An, S, red, stg);
      else bwd_item<TIO, NS, false, false>(a, j, stream, b, d, active, lane, An, S, red, stg);
    }
  }
}

}  // namespace mamba
