// scan.cuh -- selective scan kernels for sm_100a.
//
// What is computed (page "Mamba SSM Nedir? Transformer Alternatifi Rehberi
// (2026)", sections "Ayrık Zamana Geçiş" and "Mamba'nın Yeniliği: Selective
// SSM"): for every (batch b, channel d) row and state n,
//     z      = Delta[b,t,d] * A[d,n]
//     Abar   = exp(z),   Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B = (e^z - 1)/A[d,n] * B[b,t,n]
//     h[n]   = Abar h[n] + Bbar u[b,t,d]
//     y[b,t,d] = sum_n C[b,t,n] h[n] + D[d] u[b,t,d]
//
// Work decomposition
//   * A "group" is 32 consecutive channels of one batch row.  A consumer warp
//     owns a group while it runs a job, each lane one channel with its N
//     states in registers.
//   * The sequence of a group is cut into chunks.  A job is (stream, chunk):
//     a warp runs the recurrence over the chunk's tokens starting from the
//     state the previous chunk of the same stream ended with.  Jobs are
//     handed out by an atomic ticket in chunk-major order, so the predecessor
//     of every job was taken earlier by a running warp: waits always end.
//   * The grid is persistent, one CTA per SM: four consumer warps (one per SM
//     sub-partition) and one producer warp.  The producer pulls the tickets,
//     streams each consumer's tiles into its shared-memory ring by TMA and
//     publishes the consumers' chunk-to-chunk hand-off flags, so a consumer
//     only waits for a tile, computes, and hands the slot back.
//   * When there are fewer groups than consumer warps, the sequence is also
//     cut into "super-chunks" that run as independent streams, every one
//     from a zero state (super-chunk 0 from the initial state), with no wait
//     between them.  Each records its end state H_j and its sum of Delta.
//     The states entering the super-chunks then follow from the associative
//     combine of the page's parallel prefix scan ("Paralel Tarama
//     Algoritması"), h_in(j+1) = exp(A sum Delta_j) h_in(j) + H_j, and a
//     second kernel adds their effect to the outputs:
//         y_t += sum_n C_t[n] exp(A_n cum_t) h_in[n],
//     cum_t the sum of Delta from the super-chunk's start through t.  It
//     walks each super-chunk only while the slowest decay exp(A_n cum_t) is
//     at least 2^-s, s = fix_stop_log2: past that every term is below 2^-s
//     of |C_t[n] h_in[n]|.  s = 32 for fp32 data (256 times under the fp32
//     rounding of y), 20 for bf16 data (2^11 times under the bf16 rounding
//     of y).  It also writes the final state H + exp(A sum Delta) h_in of
//     the last super-chunk (exactly, not truncated).
//
// Arithmetic per token and state (all fp32; the state is kept scaled,
// g_n = A_n h_n, so that 1/A_n leaves the inner loop):
//     e_n  = expm1(Delta A_n)
//     g_n <- g_n + e_n (g_n + B_n x)          (== Abar g + e B x)
//     y   += (C_n / A_n) g_n
// When A[d,n] == (n+1) A[d,0] for every n of every channel in the warp (the
// S4D-real structure), e_n comes from one exact-arithmetic identity,
//     e^{(n+1) z} - 1 = e^z (e^{n z} - 1) + (e^z - 1),
// i.e. e_n = r e_{n-1} + q with r = exp(Delta A[d,0]), q = r - 1: one FMA per
// state instead of an exponential; then C_n / A_n = (C_n / (n+1)) / A_0.
// Otherwise every e_n is computed from its own exponential.
//
// Data path of a tile: u, Delta and B in the I/O type, and C' = C / (n+1) as
// fp32 (a small pre-pass per call), staged by TMA.  With bf16 data the input
// term B_n x is one mixed-precision FMA on the raw bf16 operands (their
// product is exact in fp32); nothing is converted in shared memory.  Every
// lane reads the whole B and C' row of every token (broadcast loads).  y is
// stored by each lane with a predicated store: no branch inside the token
// loop, which keeps a tile's tokens in one scheduling region.
#pragma once

#include "common.cuh"

namespace mamba {

#ifndef MAMBA_SCAN_PIPE
#define MAMBA_SCAN_PIPE 0
#endif
#ifndef MAMBA_SCAN_UNROLL
#define MAMBA_SCAN_UNROLL 4
#endif
constexpr int kScanUnroll = MAMBA_SCAN_UNROLL;  // token pairs per unrolled step of a full tile

constexpr int kCPW = 32;   // channels per warp: one lane per channel
constexpr int kFixSegTiles = 1;  // tiles per segment of the super-chunk correction
// the correction stops where the carried decay is below 2^-fix_stop_log2
template <typename TIO>
__host__ __device__ constexpr float fix_stop_log2() { return sizeof(TIO) == 2 ? 20.0f : 32.0f; }
constexpr int kHandQ = 8;  // hand-off flags a consumer may leave for the producer to publish

enum Discretisation : int { kZOH = 0, kEuler = 1, kTrapezoid = 2 };

struct ScanParams {
  // tensors
  const void* u;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;            // C in the I/O type [batch*len][N] (read by the correction kernel)
  const float* cs;          // C' = C / (n+1), fp32 [batch*len][N] (scratch, written by the pre-pass)
  const float4* chan;       // per channel {A[d,0], 1/A[d,0], D[d], structured}, padded to groups_d*32
  const float* h0;          // nullable: initial state [b][d][n]
  void* y;                  // nullable: no output (checkpoint-only runs for the backward)
  float* final_state;       // nullable
  float* ckpt;              // [batch][ceil(len/TILE)][channels][N] state before every tile (CKPT kernels)
  // scratch (stream-ordered; the pre-pass zeroes counters and done)
  int* counters;            // [0] job ticket, [1] abort flag
  int* done;                // [S*G] chunks completed per stream
  float* ring;              // [S*G][2][32][N] states handed between chunks
  float* ring_sd;           // [S*G][2][32] running sum of Delta in the super-chunk
  float* agg_h;             // [S*G][32][N] end state of each super-chunk (S > 1)
  float* agg_sd;            // [S*G][32]    sum of Delta over each super-chunk (S > 1)
  float* cum;               // [S*G][segs_max][32] sum of Delta before each correction segment (S > 1)
  int* fix_segs;            // [S*G] segments of the stream the correction kernel must walk (zeroed)
  // sizes
  int64_t batch, len, channels;
  int groups_d;             // ceil(channels / 32)
  int groups;               // batch * groups_d
  int supers;               // S
  int64_t super_len;        // tokens per super-chunk (all but the last)
  int64_t chunk_len;        // tokens per chunk
  int chunks_full;          // chunks of a full super-chunk
  int chunks_last;          // chunks of the last super-chunk
  int streams;              // S*G streams, stream = super * groups + group
  int segs_max;             // correction segments (kFixSegTiles tiles each) of a full super-chunk
  int fix_vec;              // Delta, y and C rows can be staged in 16-byte pieces
  int jobs;                 // all jobs (fits int32, checked on the host)
  int use_tma;
  uint64_t wait_limit_ns;
};

// ---------------------------------------------------------------------------
// job bookkeeping
// ---------------------------------------------------------------------------
struct Job {
  int stream;      // super * groups + group
  int chunk;       // chunk index inside the stream
  int b, d0;       // batch row and first channel of the group
  int64_t t0, t1;  // token range [t0, t1) of this job
  int ntiles;
  bool first, last;  // first / last chunk of the stream
  int super_idx;
};

// Tickets in chunk-major order: chunk k of every stream before chunk k+1 of
// any (the last super-chunk may have fewer chunks than the others).
__device__ __forceinline__ Job decode_job(const ScanParams& p, int j_in, int tile) {
  // 32-bit arithmetic: the host guarantees jobs, streams and b*len fit in int32
  Job jb;
  const uint32_t j = (uint32_t)j_in;
  const uint32_t n_all = (uint32_t)p.streams;
  const uint32_t n_full = (uint32_t)(p.supers - 1) * (uint32_t)p.groups;
  const uint32_t kmin = (uint32_t)p.chunks_last;
  uint32_t k, s;
  if (j < kmin * n_all) {
    k = j / n_all;
    s = j - k * n_all;
  } else {
    const uint32_t jj = j - kmin * n_all;
    const uint32_t kk = jj / n_full;
    k = kmin + kk;
    s = jj - kk * n_full;
  }
  jb.stream = (int)s;
  jb.chunk = (int)k;
  jb.super_idx = (int)(s / (uint32_t)p.groups);
  const int grp = (int)(s - (uint32_t)jb.super_idx * (uint32_t)p.groups);
  jb.b = grp / p.groups_d;
  jb.d0 = (grp - jb.b * p.groups_d) * kCPW;
  const int64_t s_begin = (int64_t)jb.super_idx * p.super_len;
  const int64_t s_end = (s_begin + p.super_len < p.len) ? s_begin + p.super_len : p.len;
  jb.t0 = s_begin + (int64_t)k * p.chunk_len;
  jb.t1 = (jb.t0 + p.chunk_len < s_end) ? jb.t0 + p.chunk_len : s_end;
  jb.ntiles = (int)((jb.t1 - jb.t0 + tile - 1) / tile);
  jb.first = (k == 0);
  jb.last = (jb.t1 == s_end);
  return jb;
}

// ---------------------------------------------------------------------------
// shared-memory block of one consumer warp: STAGES tile slots (TMA
// destinations, 128-byte aligned) with the per-channel constants of the
// job, full / empty barriers, the job of each slot, and the queue of
// hand-off flags the producer publishes
// ---------------------------------------------------------------------------
// B and C' rows are fp32 whatever the I/O type (for bf16 data the pre-pass
// widens B; the widening is exact), so the input term of every state step
// is a packed FFMA2.  R > 1 (multi-input multi-output): a token has R rows
// of u, B and C' (input / output r of row t at row t R + r) and one row of
// Delta.
template <typename TIO, int NS, int TILE, int STAGES, int R = 1>
struct alignas(128) WarpSmem {
  TIO u[STAGES][TILE * R][kCPW];
  TIO dl[STAGES][TILE][kCPW];
  float b[STAGES][TILE * R][NS];
  float cs[STAGES][TILE * R][NS];
  float4 chan[STAGES][kCPW];  // loaded with tile 0 of a job
  uint64_t full[STAGES];      // producer -> consumer: the tile has landed
  uint64_t empty[STAGES];     // consumer -> producer: the slot has been read
  int job[STAGES];            // job of the slot's tile; -1: no more jobs
  int* hq_flag[kHandQ];       // hand-off flags: *flag = value
  int hq_value[kHandQ];
  int hq_head;                // entries pushed by the consumer
  int hq_tail;                // entries published by the producer
  int finished;               // the consumer has left its loop
};

template <typename TIO, int NS, int TILE, int STAGES, int CW, int R = 1>
constexpr size_t scan_smem_bytes() {
  return sizeof(WarpSmem<TIO, NS, TILE, STAGES, R>) * CW + 128;
}

// bytes one tile brings in: u and Delta columns (I/O type), the B and C' rows (fp32)
template <typename TIO, int NS, int R = 1>
__host__ __device__ constexpr uint32_t tile_bytes(int tile) {
  return (uint32_t)(tile * ((R + 1) * kCPW * sizeof(TIO) + 2 * R * NS * sizeof(float)));
}

// ---------------------------------------------------------------------------
// per-token arithmetic
// ---------------------------------------------------------------------------
// e^z - 1 for z <= 0 without a branch: for |z| <= 1/4 the Taylor polynomial
// through z^6 in Estrin form (truncation below 1.2e-8 relative there, three
// dependent FMAs); otherwise the hardware exp2 minus one (|e^z - 1| > 0.22
// there, so its absolute error is small relative to the result).  Both are
// evaluated and one is selected.
__device__ __forceinline__ float expm1_small(float z) {
  const float z2 = z * z;
  const float lo = fmaf(z, 1.0f / 6.0f, 0.5f);                                      // 1/2 + z/6
  const float hi = fmaf(z2, 1.0f / 720.0f, fmaf(z, 1.0f / 120.0f, 1.0f / 24.0f));  // 1/24 + z/120 + z^2/720
  const float z4 = z2 * z2;
  const float poly = fmaf(z4, hi, fmaf(z2, lo, z));
  const float viaexp2 = ex2_approx(z * 1.4426950408889634f) - 1.0f;
  return fabsf(z) <= 0.25f ? poly : viaexp2;
}

// expm1_small's q = e^z - 1 together with d = q - z, both accurate to fp32
// relative precision: for |z| <= 1/4 d is the polynomial without its
// leading z (no cancellation); above, q - z does not cancel much.
__device__ __forceinline__ void expm1_parts(float z, float& q, float& d) {
  const float z2 = z * z;
  const float lo = fmaf(z, 1.0f / 6.0f, 0.5f);
  const float hi = fmaf(z2, 1.0f / 720.0f, fmaf(z, 1.0f / 120.0f, 1.0f / 24.0f));
  const float z4 = z2 * z2;
  const float dpoly = fmaf(z4, hi, z2 * lo);
  const float qexp = ex2_approx(z * 1.4426950408889634f) - 1.0f;
  const bool small = fabsf(z) <= 0.25f;
  q = small ? z + dpoly : qexp;
  d = small ? dpoly : qexp - z;
}

// exp(z) - 1 for z <= 0 without a branch, for bf16 data: the hardware exp2
// minus one (absolute error about 2.4e-7, so below 7.7e-6 relative once
// |z| >= 1/32), and for |z| < 1/32 the series z + z^2/2 + z^3/6 (truncation
// below 1.3e-6 relative there).  Both are evaluated and one is selected.
__device__ __forceinline__ float expm1_series3(float z) { return z * fmaf(z, fmaf(z, 1.0f / 6.0f, 0.5f), 1.0f); }
// the same series for z = zl ln 2 given zl (base-2 units): zl (c1 + zl (c2 + zl c3))
// with c1 = ln 2, c2 = (ln 2)^2 / 2, c3 = (ln 2)^3 / 6; |zl| < kSeriesLimit2 is |z| < 1/32
constexpr float kSeriesLimit2 = 0.03125f * 1.4426950408889634f;
__device__ __forceinline__ float expm1_series3_log2(float zl) {
  return zl * fmaf(zl, fmaf(zl, 0.0555041086648216f, 0.2402265069591007f), 0.6931471805599453f);
}
__device__ __forceinline__ float expm1_fast(float z) {
  const float viaexp2 = ex2_approx(z * 1.4426950408889634f) - 1.0f;
  return fabsf(z) < 0.03125f ? expm1_series3(z) : viaexp2;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ uint16_t raw16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }

// 16-byte asynchronous copy global -> shared; with in == false nothing is
// read and the 16 bytes are zero-filled
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool in) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(in ? 16 : 0) : "memory");
}

// Store v at p when pred holds, as one predicated instruction (a branch
// around a plain store would split the token loop into scheduling regions).
__device__ __forceinline__ void st_global_pred(__nv_bfloat16* p, __nv_bfloat16 v, bool pred) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.b16 [%0], %1;\n\t}" ::"l"(p),
               "h"(raw16(v)), "r"((int)pred));
}
__device__ __forceinline__ void st_global_pred(float* p, float v, bool pred) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.f32 [%0], %1;\n\t}" ::"l"(p),
               "f"(v), "r"((int)pred));
}

// e2[k] = (exp((2k+1) z) - 1, exp((2k+2) z) - 1) for k < NS/2 from
// r = exp(z) and q = exp(z) - 1, using
//     exp((m+k) z) - 1 = (exp(k z) - 1) + exp(k z)(exp(m z) - 1):
// the first four by steps of z, the rest by steps of 4z in four independent
// chains (dependency depth 7 instead of NS - 1).
template <int NS>
__device__ __forceinline__ void decay_chain(float r, float q, float2 (&e2)[NS / 2]) {
  static_assert(NS % 4 == 0, "NS multiple of 4");
  const float e1 = fmaf(r, q, q);
  const float e2s = fmaf(r, e1, q);
  const float e3 = fmaf(r, e2s, q);
  e2[0] = f2(q, e1);
  e2[1] = f2(e2s, e3);
  const float2 r4 = f2(1.0f + e3, 1.0f + e3);
  const float2 q4 = f2(e3, e3);
#pragma unroll
  for (int k = 2; k < NS / 2; ++k) e2[k] = __ffma2_rn(r4, e2[k - 2], q4);
}

// One token for one lane: g <- g + e (g + B x) for all states; returns
// sum_n C'_n g_n (Y; without Y, only the state steps: the checkpointing pass
// of the backward writes no output).  States as N/2 float2 pairs, every step
// a packed FFMA2 (B x is exact in fp32 for bf16 operands, so this equals the
// mixed-precision product of the raw bf16 values).
template <typename TIO, int NS, bool Y = true>
__device__ __forceinline__ float token_update(const float2 (&e)[NS / 2], const float* brow, const float* csrow, TIO xr,
                                              float2 (&g)[NS / 2]) {
  float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
  const float x = to_f32(xr);
  const float2 x2 = f2(x, x);
#pragma unroll
  for (int n4 = 0; n4 < NS / 4; ++n4) {
    const float4 bv = reinterpret_cast<const float4*>(brow)[n4];
    const int p0 = 2 * n4, p1 = 2 * n4 + 1;
    const float2 v0 = __ffma2_rn(f2(bv.x, bv.y), x2, g[p0]);
    const float2 v1 = __ffma2_rn(f2(bv.z, bv.w), x2, g[p1]);
    g[p0] = __ffma2_rn(e[p0], v0, g[p0]);
    g[p1] = __ffma2_rn(e[p1], v1, g[p1]);
    if constexpr (Y) {
      const float4 cv = reinterpret_cast<const float4*>(csrow)[n4];
      acc0 = __ffma2_rn(f2(cv.x, cv.y), g[p0], acc0);
      acc1 = __ffma2_rn(f2(cv.z, cv.w), g[p1], acc1);
    }
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// Rows [0, rows) of one tile, structured A, for one lane: its channel column
// `su`/`sdl` (stride 32) and all its states.  Stores y (predicated on the
// channel being inside the tensor) and accumulates sum(Delta) in sd.
// FASTQ (bf16 data): r from the hardware exp2 of Delta A_0 log2(e), q = r - 1
// (a short series for |Delta A_0| < 1/32); otherwise q from the accurate
// expm1 and r = 1 + q.  Two tokens per step:
// their decay chains are independent work for the scheduler while the state
// updates wait on each other.
template <typename TIO, int NS, int TILE, bool FASTQ, bool Y = true>
__device__ __forceinline__ void tile_structured(const TIO* su, const TIO* sdl, const float (*bt)[NS],
                                                const float (*ct)[NS], int rows, float a0, float inv_a0, float Dd,
                                                float2 (&g)[NS / 2], float& sd, TIO* yp, int64_t ystride,
                                                bool active) {
  const float a0l = a0 * 1.4426950408889634f;
  auto chain = [&](float dt, float2 (&e)[NS / 2]) {
    if constexpr (FASTQ) {
      // r from the hardware exp2; q = r - 1 from the same value, or from the
      // series where that subtraction would lose the small |Delta A_0|
      const float zl = dt * a0l;
      const float r = ex2_approx(zl);
      const float q = fabsf(zl) < kSeriesLimit2 ? expm1_series3_log2(zl) : r - 1.0f;
      decay_chain<NS>(r, q, e);
    } else {
      const float q = expm1_small(dt * a0);
      decay_chain<NS>(1.0f + q, q, e);
    }
  };
  auto emit = [&](float s, TIO xr, float dt) {
    if constexpr (Y) {
      st_global_pred(yp, from_f32<TIO>(fmaf(s, inv_a0, Dd * to_f32(xr))), active);
      yp += ystride;
    }
    sd += dt;
  };
  auto pair = [&](int r) {
    const TIO x0 = su[r * kCPW], x1 = su[(r + 1) * kCPW];
    const float d0 = to_f32(sdl[r * kCPW]), d1 = to_f32(sdl[(r + 1) * kCPW]);
    float2 e0[NS / 2], e1[NS / 2];
    chain(d0, e0);
    chain(d1, e1);
    const float s0 = token_update<TIO, NS, Y>(e0, bt[r], ct[r], x0, g);
    const float s1 = token_update<TIO, NS, Y>(e1, bt[r + 1], ct[r + 1], x1, g);
    emit(s0, x0, d0);
    emit(s1, x1, d1);
  };
  int r = 0;
  if (rows == TILE) {
#if MAMBA_SCAN_PIPE
    // software pipeline over token pairs: the loads and decay chains of
    // pair k+1 are issued before the state updates of pair k, so their
    // latency (shared-memory loads, exp2) overlaps the updates
    float2 ea[NS / 2], eb[NS / 2];
    TIO xa = su[0], xb = su[kCPW];
    float da = to_f32(sdl[0]), db = to_f32(sdl[kCPW]);
    chain(da, ea);
    chain(db, eb);
#pragma unroll 2
    for (; r < TILE; r += 2) {
      float2 na[NS / 2], nb[NS / 2];
      TIO nxa = xa, nxb = xb;
      float nda = 0.0f, ndb = 0.0f;
      if (r + 2 < TILE) {
        nxa = su[(r + 2) * kCPW];
        nxb = su[(r + 3) * kCPW];
        nda = to_f32(sdl[(r + 2) * kCPW]);
        ndb = to_f32(sdl[(r + 3) * kCPW]);
        chain(nda, na);
        chain(ndb, nb);
      }
      const float s0 = token_update<TIO, NS, Y>(ea, bt[r], ct[r], xa, g);
      const float s1 = token_update<TIO, NS, Y>(eb, bt[r + 1], ct[r + 1], xb, g);
      emit(s0, xa, da);
      emit(s1, xb, db);
#pragma unroll
      for (int k = 0; k < NS / 2; ++k) {
        ea[k] = na[k];
        eb[k] = nb[k];
      }
      xa = nxa;
      xb = nxb;
      da = nda;
      db = ndb;
    }
#else
#pragma unroll kScanUnroll
    for (; r < TILE; r += 2) pair(r);
#endif
  } else {
    for (; r + 1 < rows; r += 2) pair(r);
    if (r < rows) {
      const TIO x0 = su[r * kCPW];
      const float d0 = to_f32(sdl[r * kCPW]);
      float2 e0[NS / 2];
      chain(d0, e0);
      emit(token_update<TIO, NS, Y>(e0, bt[r], ct[r], x0, g), x0, d0);
    }
  }
}

// Rows [0, rows) of one tile, general A: one exponential per state.
// kA[n] = A_n log2(e), kC[n] = (n+1) / A_n (so that C'_n kC[n] = C_n / A_n).
// METHOD selects the discretisation (the state is kept scaled, g_n = A_n h_n,
// z_n = Delta A_n, e_n = exp(z_n) - 1, v_n = B_n x):
//   kZOH        g <- g + e (g + v)                        (zero-order hold)
//   kEuler      g <- (1 + e) g + z v                      (Bbar = Delta B)
//   kTrapezoid  g <- (1 + e)(g + z/2 vp) + z/2 v,  vp = the previous token's v
// (Mamba-3 page, "Geliştirilmiş Ayrıklaştırma Şeması", with the readings
// given in the header).  vp carries the previous token's v across tiles.
template <typename TIO, int NS, int METHOD>
__device__ __forceinline__ void tile_general(const TIO* su, const TIO* sdl, const float (*bt)[NS],
                                             const float (*ct)[NS], int rows, const float (&kA)[NS],
                                             const float (&kC)[NS], float Dd, float2 (&g)[NS / 2], float& sd,
                                             float (&vp)[NS], TIO* yp, int64_t ystride, bool active) {
  for (int r = 0; r < rows; ++r) {
    const TIO xr = su[r * kCPW];
    const float dt = to_f32(sdl[r * kCPW]);
    float ev[NS], zv[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
      zv[k] = dt * (kA[k] * 0.69314718055994531f);  // Delta A_n
      if constexpr (sizeof(TIO) == 4) ev[k] = expm1_small(zv[k]);  // fp32 data: accurate expm1
      else ev[k] = expm1_fast(zv[k]);
    }
    float crow[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) crow[k] = ct[r][k] * kC[k];
    float s;
    if constexpr (METHOD == kZOH) {
      float2 e[NS / 2];
#pragma unroll
      for (int k = 0; k < NS / 2; ++k) e[k] = f2(ev[2 * k], ev[2 * k + 1]);
      s = token_update<TIO, NS>(e, bt[r], crow, xr, g);
    } else {
      const float x = to_f32(xr);
      s = 0.0f;
#pragma unroll
      for (int k = 0; k < NS; ++k) {
        const float v = bt[r][k] * x;  // exact for bf16 operands
        float gk = (k & 1) ? g[k >> 1].y : g[k >> 1].x;
        if constexpr (METHOD == kEuler) {
          gk = fmaf(ev[k], gk, fmaf(zv[k], v, gk));
        } else {
          const float zh = 0.5f * zv[k];
          gk = fmaf(1.0f + ev[k], fmaf(zh, vp[k], gk), zh * v);
          vp[k] = v;
        }
        if (k & 1) g[k >> 1].y = gk;
        else g[k >> 1].x = gk;
        s = fmaf(crow[k], gk, s);
      }
    }
    st_global_pred(yp, from_f32<TIO>(s + Dd * to_f32(xr)), active);
    yp += ystride;
    sd += dt;
  }
}

// ---------------------------------------------------------------------------
// Multi-input multi-output (R > 1; the Mamba-3 page, "MIMO Mekanizmasının
// İşleyişi", read as: R inputs and R outputs per channel share one state and
// one step).  One token for one lane:
//     g_n <- g_n + e_n (g_n + sum_r B^(r)_n x^(r))        (one state update)
//     acc[r] = sum_n C'^(r)_n g_n                          (R outputs, each
//                                                          with its own gate C^(r))
// brows / csrows: the token's R rows of B and C'; xs: the lane's x^(0) with
// x^(r) at xs[r * 32].  GEN: general A, C'^(r)_n is scaled by kC[n].
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int R, bool GEN>
__device__ __forceinline__ void token_update_mimo(const float2 (&e)[NS / 2], const float* brows, const float* csrows,
                                                  const TIO* xs, const float (&kC)[GEN ? NS : 1],
                                                  float2 (&g)[NS / 2], float (&acc)[R]) {
  static_assert(NS % 8 == 0, "MIMO rows are read in 16-byte pieces");
  float2 a2[R];
#pragma unroll
  for (int r = 0; r < R; ++r) a2[r] = f2(0.f, 0.f);
  float2 v[NS / 2];
#pragma unroll
  for (int k = 0; k < NS / 2; ++k) v[k] = g[k];
  // input terms: sum over r of B^(r) x^(r), added to g
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float x = to_f32(xs[r * kCPW]);
    const float2 x2 = f2(x, x);
#pragma unroll
    for (int k4 = 0; k4 < NS / 4; ++k4) {
      const float4 bv = reinterpret_cast<const float4*>(brows + r * NS)[k4];
      v[2 * k4] = __ffma2_rn(f2(bv.x, bv.y), x2, v[2 * k4]);
      v[2 * k4 + 1] = __ffma2_rn(f2(bv.z, bv.w), x2, v[2 * k4 + 1]);
    }
  }
#pragma unroll
  for (int k = 0; k < NS / 2; ++k) g[k] = __ffma2_rn(e[k], v[k], g[k]);
  // outputs
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int k4 = 0; k4 < NS / 4; ++k4) {
      float4 cv = reinterpret_cast<const float4*>(csrows + r * NS)[k4];
      if constexpr (GEN) {
        cv.x *= kC[4 * k4]; cv.y *= kC[4 * k4 + 1]; cv.z *= kC[4 * k4 + 2]; cv.w *= kC[4 * k4 + 3];
      }
      a2[r] = __ffma2_rn(f2(cv.x, cv.y), g[2 * k4], a2[r]);
      a2[r] = __ffma2_rn(f2(cv.z, cv.w), g[2 * k4 + 1], a2[r]);
    }
    acc[r] = a2[r].x + a2[r].y;
  }
}

// Rows [0, rows) of one multi-input multi-output tile for one lane (tokens
// of the tile; token r has u rows r R .. r R + R-1).  STRUCT: the decays
// from the decay chain; otherwise one exponential per state (kA = A log2 e,
// kC = (n+1)/A_n).  Stores the R outputs of each token (predicated) and
// accumulates sum(Delta) in sd.  y of token t, output q, sits at
// yp + (t R + q) ystride.
template <typename TIO, int NS, int R, bool STRUCT, bool FASTQ>
__device__ __forceinline__ void tile_mimo(const TIO* su, const TIO* sdl, const float (*bt)[NS], const float (*ct)[NS],
                                          int rows, float a0, float inv_a0, const float (&kA)[STRUCT ? 1 : NS],
                                          const float (&kC)[STRUCT ? 1 : NS], float Dd, float2 (&g)[NS / 2],
                                          float& sd, TIO* yp, int64_t ystride, bool active) {
  const float a0l = a0 * 1.4426950408889634f;
#pragma unroll 2
  for (int r = 0; r < rows; ++r) {
    const float dt = to_f32(sdl[r * kCPW]);
    float2 e[NS / 2];
    if constexpr (STRUCT) {
      if constexpr (FASTQ) {
        const float zl = dt * a0l;
        const float rr = ex2_approx(zl);
        decay_chain<NS>(rr, fabsf(zl) < kSeriesLimit2 ? expm1_series3_log2(zl) : rr - 1.0f, e);
      } else {
        const float q = expm1_small(dt * a0);
        decay_chain<NS>(1.0f + q, q, e);
      }
    } else {
#pragma unroll
      for (int k = 0; k < NS / 2; ++k) {
        const float z0 = dt * (kA[2 * k] * 0.69314718055994531f), z1 = dt * (kA[2 * k + 1] * 0.69314718055994531f);
        e[k] = sizeof(TIO) == 4 ? f2(expm1_small(z0), expm1_small(z1)) : f2(expm1_fast(z0), expm1_fast(z1));
      }
    }
    float acc[R];
    token_update_mimo<TIO, NS, R, !STRUCT>(e, bt[r * R], ct[r * R], su + r * R * kCPW, kC, g, acc);
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const float xq = to_f32(su[(r * R + q) * kCPW]);
      const float yq = STRUCT ? fmaf(acc[q], inv_a0, Dd * xq) : fmaf(Dd, xq, acc[q]);
      st_global_pred(yp + q * ystride, from_f32<TIO>(yq), active);
    }
    yp += R * ystride;
    sd += dt;
  }
}

// ---------------------------------------------------------------------------
// consumer side of one warp's tile pipeline
// ---------------------------------------------------------------------------
__device__ __forceinline__ void abort_scan(const ScanParams& p) {
  record_device_error(MAMBA_ERR_TIMEOUT);
  atomicExch(&p.counters[1], 1);
}

template <typename TIO, int NS, int TILE, int STAGES, int R = 1>
struct Consumer {
  using Smem = WarpSmem<TIO, NS, TILE, STAGES, R>;
  const ScanParams& p;
  Smem& sm;
  int lane;
  uint32_t seq = 0;  // tiles consumed
  int hq_head = 0;   // lane 0: hand-off entries pushed

  __device__ Consumer(const ScanParams& p_, Smem& sm_, int lane_) : p(p_), sm(sm_), lane(lane_) {}

  // wait for the next tile; its slot, or -1 when the wait gave up
  __device__ int wait_tile() {
    const int s = seq % STAGES;
    bool ok = mbar_wait_bounded(&sm.full[s], (seq / STAGES) & 1u, p.wait_limit_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) abort_scan(p);
      return -1;
    }
    return s;
  }

  // the tile is read: hand its slot back to the producer
  __device__ void release_tile() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[seq % STAGES]);
    ++seq;
  }

  // without TMA the warp fetches its tile itself (rows of this job only)
  __device__ void fetch_tile(int s, const Job& jb, int64_t tt0, int rows, int d, bool active) {
    const TIO* gu = static_cast<const TIO*>(p.u);
    const TIO* gdl = static_cast<const TIO*>(p.delta);
    const TIO* gB = static_cast<const TIO*>(p.B);
    const int64_t rowbase = (int64_t)jb.b * p.len + tt0;
    for (int r = 0; r < rows; ++r) {
      const int64_t off = (rowbase + r) * p.channels + d;
      sm.dl[s][r][lane] = active ? gdl[off] : from_f32<TIO>(0.0f);
    }
    for (int r = 0; r < rows * R; ++r) {
      const int64_t off = (rowbase * R + r) * p.channels + d;
      sm.u[s][r][lane] = active ? gu[off] : from_f32<TIO>(0.0f);
    }
    for (int i = lane; i < rows * R * NS; i += 32) {
      const int r = i / NS, n = i - r * NS;
      sm.b[s][r][n] = to_f32(gB[(rowbase * R + r) * NS + n]);
      sm.cs[s][r][n] = p.cs[(rowbase * R + r) * NS + n];
    }
    __syncwarp();
  }

  // wait until *flag >= target (the previous chunk of the stream has handed
  // its state on).  The limit counts time without progress of the whole
  // grid: the deadline restarts whenever the job ticket moves.
  __device__ bool wait_flag(const int* flag, int target) {
    bool aborted = false;
    if (lane == 0) {
      uint64_t t_start = globaltimer_ns();
      int ticket = ld_volatile(&p.counters[0]);
      uint32_t spins = 0;
      while (ld_acquire(flag) < target) {
        if (ld_volatile(&p.counters[1]) != 0) { aborted = true; break; }
        if ((++spins & 31u) == 0) {
          const uint64_t now = globaltimer_ns();
          const int t = ld_volatile(&p.counters[0]);
          if (t != ticket) {
            ticket = t;
            t_start = now;
          } else if (now - t_start > p.wait_limit_ns) {
            abort_scan(p);
            aborted = true;
            break;
          }
        }
        __nanosleep(spins < 64 ? 32 : 256);
      }
    }
    // lane 0's acquire, then the warp barrier, orders the state reads below
    // after the predecessor's release; they bypass L1 (ld.cg) so no stale
    // line of an earlier chunk can be hit
    aborted = __shfl_sync(0xffffffffu, (int)aborted, 0) != 0;
    return !aborted;
  }

  // Lane 0, after a __syncwarp that follows every lane's state stores:
  // *flag = value.  The producer warp publishes it (its gpu-scope release
  // covers the stores, which it observed through this cta-scope release), so
  // the consumer does not wait for the fence; if the queue is full the
  // consumer publishes it itself.
  __device__ void publish(int* flag, int value) {
    if (hq_head - ld_relaxed_cta_smem(&sm.hq_tail) < kHandQ) {
      sm.hq_flag[hq_head % kHandQ] = flag;
      sm.hq_value[hq_head % kHandQ] = value;
      ++hq_head;
      st_release_cta_smem(&sm.hq_head, hq_head);
    } else {
      st_release(flag, value);
    }
  }
};

// ---------------------------------------------------------------------------
// producer warp (lane 0): pulls jobs from the global ticket, decodes them and
// streams their tiles into every consumer's slots (TMA, or a bare arrive
// when the consumer fetches by itself); publishes the consumers' hand-off
// flags; ends each consumer's stream with a job id of -1.
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int CW, int TILE, int STAGES, int R = 1>
__device__ void producer_loop(const ScanParams& p, WarpSmem<TIO, NS, TILE, STAGES, R>* sms, const CUtensorMap* mu,
                              const CUtensorMap* mdl, const CUtensorMap* mb, const CUtensorMap* mc) {
  struct Feed {
    uint32_t seq;   // tiles (and the end mark) issued
    int job, tile, ntiles;
    int row0, d0;
    int hq_tail;    // hand-off entries published
    bool ended;     // end mark issued (or the consumer left)
    bool fin;       // the consumer has left its loop
  };
  Feed f[CW];
#pragma unroll
  for (int w = 0; w < CW; ++w) f[w] = Feed{0u, -1, 0, 0, 0, 0, 0, false, false};
  // The next job's ticket is taken when some consumer's job issues its last
  // tile (or, failing that, when a consumer needs a job), not as soon as the
  // previous one is used: a ticket held until one of this CTA's consumers
  // frees up (up to a whole job) would start its job long after the jobs of
  // the neighbouring tickets, i.e. the neighbouring channel groups that read
  // the other halves of the same 128-byte u and Delta lines, which by then
  // have left L2 (measured at 2^20 tokens x 2048 channels: 11.6 -> 8.7 GB
  // read per launch).
  int ticket = -1;
  bool stop = false;                          // some warp gave up: hand out no more jobs
  uint32_t idle = 0;
  uint64_t idle_since = 0;
  int seen_ticket = -1;
  for (;;) {
    bool progress = false, all_done = true;
#pragma unroll
    for (int w = 0; w < CW; ++w) {
      auto& sm = sms[w];
      // consumer state first, then its queue: seeing `finished` makes every
      // entry it pushed before visible to the queue read that follows
      if (!f[w].fin) f[w].fin = ld_acquire_cta_smem(&sm.finished) != 0;
      const int head = ld_acquire_cta_smem(&sm.hq_head);
      if (f[w].hq_tail != head) {
        for (; f[w].hq_tail != head; ++f[w].hq_tail) {
          const int e = f[w].hq_tail % kHandQ;
          st_release(sm.hq_flag[e], sm.hq_value[e]);
        }
        st_relaxed_cta_smem(&sm.hq_tail, f[w].hq_tail);
        progress = true;
      }
      if (f[w].fin) f[w].ended = true;  // left early (gave up): feed it no more
      if (!f[w].ended) {
        const uint32_t k = f[w].seq;
        const int s = (int)(k % STAGES);
        if (k < (uint32_t)STAGES || mbar_test_wait(&sm.empty[s], ((k / STAGES) - 1u) & 1u)) {
          bool issue = true;
          if (f[w].tile >= f[w].ntiles) {
            if (!stop && ticket < 0) ticket = atomicAdd(&p.counters[0], 1);
            if (!stop && ticket < p.jobs) {
              const Job jb = decode_job(p, ticket, TILE);
              f[w].job = ticket;
              f[w].tile = 0;
              f[w].ntiles = jb.ntiles;
              f[w].row0 = (int)(jb.b * p.len + jb.t0);
              f[w].d0 = jb.d0;
              ticket = -1;
            } else {
              sm.job[s] = -1;  // end of this consumer's work
              mbar_arrive(&sm.full[s]);
              f[w].seq = k + 1;
              f[w].ended = true;
              issue = false;
            }
          }
          if (issue) {
            sm.job[s] = f[w].job;
            if (p.use_tma) {
              const int row = f[w].row0 + f[w].tile * TILE;
              const bool first = f[w].tile == 0;
              constexpr uint32_t kChanBytes = kCPW * sizeof(float4);
              mbar_arrive_expect_tx(&sm.full[s], tile_bytes<TIO, NS, R>(TILE) + (first ? kChanBytes : 0u));
              tma_load_2d(&sm.u[s][0][0], mu, &sm.full[s], f[w].d0, row * R);
              tma_load_2d(&sm.dl[s][0][0], mdl, &sm.full[s], f[w].d0, row);
              // B and C' rows are read by every channel group of the
              // batch row: keep them in L2 ahead of the u and Delta lines
              const uint64_t keep = l2_policy_evict_last();
              tma_load_2d_hint(&sm.b[s][0][0], mb, &sm.full[s], 0, row * R, keep);
              tma_load_2d_hint(&sm.cs[s][0][0], mc, &sm.full[s], 0, row * R, keep);
              if (first) bulk_load(&sm.chan[s][0], p.chan + f[w].d0, kChanBytes, &sm.full[s]);
            } else {
              mbar_arrive(&sm.full[s]);
            }
            ++f[w].tile;
            f[w].seq = k + 1;
            if (!stop && ticket < 0 && f[w].tile >= f[w].ntiles) ticket = atomicAdd(&p.counters[0], 1);
          }
          progress = true;
        }
      }
      all_done = all_done && f[w].fin && f[w].hq_tail == head;
    }
    if (all_done) break;
    if (progress) {
      idle = 0;
      continue;
    }
    // nothing to do: back off (the consumers run on the same sub-partitions).
    // Idle time counts only while the whole grid makes no progress (the job
    // ticket does not move): this CTA's consumers may legitimately wait for
    // the chunks of other CTAs for a long time.
    const uint64_t now = globaltimer_ns();
    if (idle == 0) idle_since = now;
    ++idle;
    if ((idle & 15u) == 0) {
      if (!stop && ld_volatile(&p.counters[1]) != 0) stop = true;
      const int t = ld_volatile(&p.counters[0]);
      if (t != seen_ticket) {
        seen_ticket = t;
        idle_since = now;
      }
    }
    if (now - idle_since > 2 * p.wait_limit_ns) {  // the consumers' own limits expire first
      abort_scan(p);
      break;
    }
    __nanosleep(idle < 8 ? 64 : 256);
  }
  // every TMA load issued must land before the CTA exits: wait for the last
  // issue into each slot (a consumer that gave up may have left some unread)
#pragma unroll
  for (int w = 0; w < CW; ++w) {
    for (int s = 0; s < STAGES; ++s) {
      if ((uint32_t)s >= f[w].seq) break;
      const uint32_t k_last = f[w].seq - 1u - ((f[w].seq - 1u - (uint32_t)s) % STAGES);
      if (!mbar_wait_bounded(&sms[w].full[s], (k_last / STAGES) & 1u, p.wait_limit_ns)) {
        record_device_error(MAMBA_ERR_TIMEOUT);
        return;
      }
    }
  }
}

// One job: the recurrence over the chunk's tokens for the warp's channels,
// from the state the previous chunk handed on, then hand the end state on.
// Lane l serves channel d0 + l and all its states.  STRUCT: A[d,n] = (n+1)
// A[d,0] on every lane (see decay_chain).  Tile 0 is already in slot s0;
// cm = {A[d,0], 1/A[d,0], D[d], structured}.
template <typename TIO, int NS, int TILE, int STAGES, bool STRUCT, int METHOD = kZOH, bool CKPT = false, int R = 1>
__device__ __forceinline__ bool run_job(Consumer<TIO, NS, TILE, STAGES, R>& cx, const Job& jb, int s0,
                                        const float4 cm) {
  static_assert(!STRUCT || METHOD == kZOH, "the structured-A path is zero-order hold only");
  static_assert(R == 1 || (METHOD == kZOH && !CKPT), "multi-input multi-output: zero-order hold, forward only");
  const ScanParams& p = cx.p;
  auto& sm = cx.sm;
  const int c = cx.lane;
  const int d = jb.d0 + c;
  const bool active = d < p.channels;
  const float a0 = cm.x;
  const float Dd = cm.z;
  const float* Arow = p.A + (int64_t)(active ? d : 0) * NS;

  // the stream's slot pair in the hand-off ring and its progress flag
  int* flag = p.done + jb.stream;
  if (!jb.first && !cx.wait_flag(flag, jb.chunk)) return false;

  // starting state, kept scaled: g_n = A_n h_n; sd = sum of Delta since the
  // super-chunk's start
  float2 g[NS / 2];
  float sd = 0.0f;
  {
    float an[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
      if constexpr (STRUCT) an[k] = (float)(k + 1) * a0;
      else an[k] = active ? __ldg(Arow + k) : -1.0f;
    }
    float h[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) h[k] = 0.0f;
    if (!jb.first) {
      const int64_t slot_i = (int64_t)jb.stream * 2 + ((jb.chunk - 1) & 1);
      const float* src = p.ring + slot_i * (kCPW * NS) + c * NS;
#pragma unroll
      for (int k = 0; k < NS; ++k) h[k] = __ldcg(src + k);
      sd = __ldcg(p.ring_sd + slot_i * kCPW + c);
    } else if (jb.super_idx == 0 && p.h0 && active) {
      // the first super-chunk starts from the initial state, the others from
      // zero (the correction kernel adds what enters them)
      const float* src = p.h0 + ((int64_t)jb.b * p.channels + d) * NS;
#pragma unroll
      for (int k = 0; k < NS; ++k) h[k] = __ldcg(src + k);
    }
#pragma unroll
    for (int k = 0; k < NS / 2; ++k) g[k] = f2(h[2 * k] * an[2 * k], h[2 * k + 1] * an[2 * k + 1]);
  }
  // super-chunks 1..S-1 ran from zero: leave the correction kernel the sum
  // of Delta at every segment start, until the slowest decay falls below
  // 2^-fix_stop_log2 on every lane (the carried state's term is negligible
  // at the output's precision for the rest of the super-chunk)
  bool track = p.supers > 1 && jb.super_idx > 0;
  float kmax = 0.0f;
  if (track) {
    if constexpr (STRUCT) {
      kmax = a0 * 1.4426950408889634f;
    } else {
      float amax = active ? __ldg(Arow) : -1.0f;
#pragma unroll
      for (int k = 1; k < NS; ++k) amax = fmaxf(amax, active ? __ldg(Arow + k) : -1.0f);
      kmax = amax * 1.4426950408889634f;
    }
  }
  const int64_t tile0 = (jb.t0 - (int64_t)jb.super_idx * p.super_len) / TILE;  // tile index in the super-chunk
  float kA[STRUCT ? 1 : NS], kC[STRUCT ? 1 : NS];
  if constexpr (!STRUCT) {
#pragma unroll
    for (int k = 0; k < NS; ++k) {
      const float an = active ? __ldg(Arow + k) : -1.0f;
      kA[k] = an * 1.4426950408889634f;
      kC[k] = (float)(k + 1) / an;
    }
  }
  // trapezoid: the input term of the token before the chunk (none at t = 0)
  float vp[NS];  // used by the trapezoid only
  if constexpr (METHOD == kTrapezoid) {
    const bool has_prev = active && jb.t0 > 0;
    const int64_t prow = (int64_t)jb.b * p.len + (has_prev ? jb.t0 - 1 : 0);
    const float xprev = has_prev ? to_f32(static_cast<const TIO*>(p.u)[prow * p.channels + d]) : 0.0f;
#pragma unroll
    for (int k = 0; k < NS; ++k)
      vp[k] = has_prev ? to_f32(static_cast<const TIO*>(p.B)[prow * NS + k]) * xprev : 0.0f;
  }

  const bool store_y = active && p.y != nullptr;
  TIO* yrow = static_cast<TIO*>(p.y) + ((int64_t)jb.b * p.len + jb.t0) * R * p.channels + d;
  for (int it = 0; it < jb.ntiles; ++it) {
    const int64_t tt0 = jb.t0 + (int64_t)it * TILE;
    const int rows = (int)(jb.t1 - tt0 < (int64_t)TILE ? jb.t1 - tt0 : (int64_t)TILE);
    if (track && (tile0 + it) % kFixSegTiles == 0) {
      if (__all_sync(0xffffffffu, !active || sd * kmax < -fix_stop_log2<TIO>())) {
        track = false;
      } else {
        const int seg = (int)((tile0 + it) / kFixSegTiles);
        p.cum[((int64_t)jb.stream * p.segs_max + seg) * kCPW + c] = sd;
        if (c == 0) atomicMax(p.fix_segs + jb.stream, seg + 1);
      }
    }
    if (CKPT && active) {
      // the state before this tile, unscaled (tiles start at multiples of TILE)
      float* ck = p.ckpt + (((int64_t)jb.b * ((p.len + TILE - 1) / TILE) + tt0 / TILE) * p.channels + d) * NS;
#pragma unroll
      for (int k = 0; k < NS; ++k) {
        const float an = STRUCT ? (float)(k + 1) * a0 : __ldg(Arow + k);
        ck[k] = ((k & 1) ? g[k >> 1].y : g[k >> 1].x) / an;
      }
    }
    const int slot = it == 0 ? s0 : cx.wait_tile();
    if (slot < 0) return false;
    if (!p.use_tma) cx.fetch_tile(slot, jb, tt0, rows, d, active);
    const TIO* su = &sm.u[slot][0][c];
    const TIO* sdl = &sm.dl[slot][0][c];
    constexpr bool kFastQ = sizeof(TIO) == 2;  // bf16 data: hardware exp2 for expm1
    if constexpr (R > 1) {
      tile_mimo<TIO, NS, R, STRUCT, kFastQ>(su, sdl, sm.b[slot], sm.cs[slot], rows, a0, cm.y, kA, kC, Dd, g, sd,
                                            yrow, p.channels, store_y);
    } else if constexpr (STRUCT) {
      tile_structured<TIO, NS, TILE, kFastQ, !CKPT>(su, sdl, sm.b[slot], sm.cs[slot], rows, a0, cm.y, Dd, g, sd,
                                                    yrow, p.channels, store_y);
    } else {
      tile_general<TIO, NS, METHOD>(su, sdl, sm.b[slot], sm.cs[slot], rows, kA, kC, Dd, g, sd, vp, yrow,
                                    p.channels, store_y);
    }
    yrow += (int64_t)rows * R * p.channels;
    cx.release_tile();
  }

  // hand the end state on (unscaled): to the next chunk, or as the final
  // state, or as the super-chunk's aggregate for the correction kernel
  float* dst;
  float* dst_sd = nullptr;
  if (!jb.last) {
    const int64_t slot_i = (int64_t)jb.stream * 2 + (jb.chunk & 1);
    dst = p.ring + slot_i * (kCPW * NS) + c * NS;
    dst_sd = p.ring_sd + slot_i * kCPW + c;
  } else if (p.supers == 1) {
    dst = (p.final_state && active) ? p.final_state + ((int64_t)jb.b * p.channels + d) * NS : nullptr;
  } else {
    dst = p.agg_h + ((int64_t)jb.stream * kCPW + c) * NS;
    dst_sd = p.agg_sd + (int64_t)jb.stream * kCPW + c;
  }
  if (dst) {
#pragma unroll
    for (int k = 0; k < NS; ++k) {
      float inv;
      if constexpr (STRUCT) inv = 1.0f / ((float)(k + 1) * a0);
      else inv = active ? 1.0f / __ldg(Arow + k) : -1.0f;
      dst[k] = ((k & 1) ? g[k >> 1].y : g[k >> 1].x) * inv;
    }
  }
  if (dst_sd) *dst_sd = sd;
  if (!jb.last) {
    // the warp barrier orders every lane's state stores before lane 0's
    // hand-off, which releases them with the flag
    __syncwarp();
    if (c == 0) cx.publish(flag, jb.chunk + 1);
  }
  __syncwarp();
  return true;
}

// ---------------------------------------------------------------------------
// the persistent chunked scan kernel: CW consumer warps (one job at a time
// each) and one producer warp (index CW) per CTA; METHOD is the
// discretisation (zero-order hold, or the general-A path with exponential
// Euler or the trapezoid rule); CKPT kernels also leave the state before
// every tile in p.ckpt (for the backward)
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int CW, int TILE, int STAGES, int METHOD, bool CKPT, int R = 1>
__global__ void __launch_bounds__((CW + 1) * 32, 1)
scan_chunks_kernel(const __grid_constant__ ScanParams p, const __grid_constant__ CUtensorMap map_u,
                   const __grid_constant__ CUtensorMap map_dl, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_c) {
  using Smem = WarpSmem<TIO, NS, TILE, STAGES, R>;
  // TMA destinations must start on 128-byte boundaries
  static_assert(sizeof(Smem) % 128 == 0, "per-warp block keeps 128-byte alignment");
  static_assert((sizeof(TIO) * TILE * R * kCPW) % 128 == 0 && (sizeof(TIO) * TILE * kCPW) % 128 == 0 &&
                    (sizeof(TIO) * TILE * R * NS) % 128 == 0 && (sizeof(float) * TILE * R * NS) % 128 == 0,
                "tile slots keep 128-byte alignment");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // align to 128 bytes by pointer arithmetic (an integer round trip would
  // hide from the compiler that these are shared-memory addresses)
  unsigned char* smem_base = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  Smem* sms = reinterpret_cast<Smem*>(smem_base);

  if (threadIdx.x < CW) {
    Smem& s = sms[threadIdx.x];
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    s.hq_head = 0;
    s.hq_tail = 0;
    s.finished = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == CW * 32 && p.use_tma) {
    tma_prefetch_desc(&map_u);
    tma_prefetch_desc(&map_dl);
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_c);
  }
  // the setup above overlaps the end of the previous kernel (programmatic
  // launch); everything below reads what it wrote
  griddep_wait();
  __syncthreads();

  if (warp == CW) {
    if (lane == 0) producer_loop<TIO, NS, CW, TILE, STAGES, R>(p, sms, &map_u, &map_dl, &map_b, &map_c);
    return;
  }

  Consumer<TIO, NS, TILE, STAGES, R> cx(p, sms[warp], lane);
  for (;;) {
    const int s0 = cx.wait_tile();
    if (s0 < 0) break;
    const int j = cx.sm.job[s0];
    if (j < 0) break;  // the producer's end mark
    const Job jb = decode_job(p, j, TILE);
    const float4 cm = p.use_tma ? cx.sm.chan[s0][lane] : __ldg(p.chan + jb.d0 + lane);
    // structured A on every channel of the warp (decided per channel by the pre-pass)
    const bool structured = __all_sync(0xffffffffu, cm.w != 0.0f);
    bool ok;
    if constexpr (METHOD != kZOH)  // other discretisations: the general-A path
      ok = run_job<TIO, NS, TILE, STAGES, false, METHOD>(cx, jb, s0, cm);
    else if (structured)
      ok = run_job<TIO, NS, TILE, STAGES, true, kZOH, CKPT, R>(cx, jb, s0, cm);
    else
      ok = run_job<TIO, NS, TILE, STAGES, false, kZOH, CKPT, R>(cx, jb, s0, cm);
    if (!ok) break;
  }
  __syncwarp();
  if (lane == 0) st_release_cta_smem(&cx.sm.finished, 1);
}

// ---------------------------------------------------------------------------
// Correction of super-chunks 1..S-1 (launched only when S > 1).  The state
// entering super-chunk j is the combine of the earlier super-chunks'
// aggregates (the monoid of the page's parallel prefix scan),
//     h_in = 0;   h_in <- exp(A sum Delta_i) h_in + H_i   for i = 0 .. j-1
// (H_0 already carries the initial state).  The main pass ran super-chunk j
// from zero, so each of its outputs misses
//     sum_n C_t[n] exp(A_n cum_t) h_in[n],   cum_t = sum of Delta from the
//                                            super-chunk's start through t.
// The main pass left cum at the start of every tile, up to the tile where
// the slowest decay falls below 2^-fix_stop_log2 on every lane (from there
// on the term is below that fraction of its size), and the number of such
// tiles per stream.  One warp per (stream of a super-chunk j >= 1, phase w),
// a lane per channel, takes tiles w, w + phases, ...: it stages the tile's
// Delta and y rows and the pre-pass's fp32 C' = C / (n+1) rows in its shared
// memory (16-byte cp.async copies, all in flight at once; plain loads when
// rows are not 16-byte pieces), adds the term token by token, and writes y
// back.  With C' the carried state is taken as hs_n = (n+1) h_n, and for
// structured A the term sum_n C'_n hs_n rho^(n+1) is a Horner scheme in
// rho^2 over pairs of states (even states in one half of a packed FFMA2,
// odd ones in the other).  Phase 0 of the last super-chunk writes
// the final state H + exp(A sum Delta) h_in.  CKPT: the state checkpointed
// before every walked tile gets exp(A_n cum) h_in[n] added.
// ---------------------------------------------------------------------------
constexpr int kFixWarps = 4;
#ifndef MAMBA_FIX_PHASES
#define MAMBA_FIX_PHASES 4
#endif
// warps per stream of the correction (tiles w, w + phases, ...): a warp
// composes its entering state once and then walks several tiles (measured
// on 2048 channels, 32 / 8 / 4 / 2 phases: 2^14 tokens 0.283 / 0.273 / 0.262
// / 0.285 ms, 2^20 8.19 / 8.13 / 8.12 / 8.12 ms)
constexpr int kFixPhases = MAMBA_FIX_PHASES;

template <typename TIO, int NS, int TILE, int R>
__host__ __device__ constexpr int fix_stage_bytes() {  // one warp: Delta [TILE][32], y [TILE*R][32], C' [TILE*R][NS] fp32
  return (TILE * kCPW + TILE * R * kCPW) * (int)sizeof(TIO) + TILE * R * NS * (int)sizeof(float);
}

template <typename TIO, int NS, int TILE, bool CKPT, int R = 1>
__global__ void __launch_bounds__(kFixWarps * 32)
scan_fix_kernel(const __grid_constant__ ScanParams p, int phases) {
  extern __shared__ __align__(16) unsigned char fix_smem[];
  griddep_wait();  // the main pass's outputs, aggregates and tile sums
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int kChunk = 16 / (int)sizeof(TIO);  // elements per 16-byte piece
  const int lane = threadIdx.x & 31;
  const int wl = threadIdx.x >> 5;
  const int64_t wg = (int64_t)blockIdx.x * kFixWarps + wl;
  const int64_t fix_streams = (int64_t)(p.supers - 1) * p.groups;
  if (wg >= fix_streams * phases) return;  // whole warps: the votes below stay full
  const int si = (int)(wg / phases);
  const int w = (int)(wg - (int64_t)si * phases);
  const int stream = p.groups + si;
  const int super_idx = stream / p.groups;
  const int grp = stream - super_idx * p.groups;
  const int b = grp / p.groups_d;
  const int d0 = (grp - b * p.groups_d) * kCPW;
  const int d = d0 + lane;
  const bool active = d < p.channels;
  const float4 cm = __ldg(p.chan + d0 + lane);
  const bool structured = __all_sync(0xffffffffu, cm.w != 0.0f);
  float an[NS];
#pragma unroll
  for (int k = 0; k < NS; ++k)
    an[k] = structured ? (float)(k + 1) * cm.x : (active ? __ldg(p.A + (int64_t)d * NS + k) : -1.0f);

  // exp(A_n sd) for every state: one exponential and a product chain when
  // A is structured (exp((n+1) A_0 sd) = exp(A_0 sd)^(n+1)), else one each
  auto decays = [&](float sd, float (&e)[NS]) {
    if (structured) {
      const float r = ex2_approx(sd * an[0] * kLog2e);
      e[0] = r;
#pragma unroll
      for (int k = 1; k < NS; ++k) e[k] = e[k - 1] * r;
    } else {
#pragma unroll
      for (int k = 0; k < NS; ++k) e[k] = ex2_approx(sd * an[k] * kLog2e);
    }
  };
  // the entering state: h <- exp(A sum Delta_j) h + H_j over the earlier
  // super-chunks (the loads of a step do not wait for the previous step)
  float h[NS];
#pragma unroll
  for (int k = 0; k < NS; ++k) h[k] = 0.0f;
#pragma unroll 2
  for (int j = 0; j < super_idx; ++j) {
    const int64_t sj = (int64_t)j * p.groups + grp;
    const float sdj = __ldcg(p.agg_sd + sj * kCPW + lane);
    const float4* H = reinterpret_cast<const float4*>(p.agg_h + (sj * kCPW + lane) * NS);
    float e[NS];
    decays(sdj, e);
#pragma unroll
    for (int k = 0; k < NS / 4; ++k) {
      const float4 v = __ldcg(H + k);
      h[4 * k] = fmaf(e[4 * k], h[4 * k], v.x);
      h[4 * k + 1] = fmaf(e[4 * k + 1], h[4 * k + 1], v.y);
      h[4 * k + 2] = fmaf(e[4 * k + 2], h[4 * k + 2], v.z);
      h[4 * k + 3] = fmaf(e[4 * k + 3], h[4 * k + 3], v.w);
    }
  }
  if (super_idx == p.supers - 1 && w == 0 && p.final_state && active) {
    const float sdl = __ldcg(p.agg_sd + (int64_t)stream * kCPW + lane);
    const float* H = p.agg_h + ((int64_t)stream * kCPW + lane) * NS;
    float* dst = p.final_state + ((int64_t)b * p.channels + d) * NS;
    float e[NS];
    decays(sdl, e);
#pragma unroll
    for (int k = 0; k < NS; ++k) dst[k] = fmaf(e[k], h[k], __ldcg(H + k));
  }

  const float a0l = cm.x * kLog2e;  // structured: every decay is a power of exp(A_0 cum)
  float kmax = an[0];  // the slowest decay of the lane
#pragma unroll
  for (int k = 1; k < NS; ++k) kmax = fmaxf(kmax, an[k]);
  kmax *= kLog2e;
  const int64_t s_begin = (int64_t)super_idx * p.super_len;
  const int64_t s_end = (s_begin + p.super_len < p.len) ? s_begin + p.super_len : p.len;
  const int tiles = ld_volatile(p.fix_segs + stream);
  const TIO* dl = static_cast<const TIO*>(p.delta);
  const float* Cs = p.cs;  // C' = C / (n+1), fp32
  TIO* y = static_cast<TIO*>(p.y);
  // this warp's staging area
  TIO* sdl = reinterpret_cast<TIO*>(fix_smem + wl * fix_stage_bytes<TIO, NS, TILE, R>());  // [TILE][32]
  TIO* sy = sdl + TILE * kCPW;                                                              // [TILE*R][32]
  float* sc = reinterpret_cast<float*>(sy + TILE * R * kCPW);                               // [TILE*R][NS]
  const uint32_t s_dl = smem_addr(sdl), s_y = smem_addr(sy), s_c = smem_addr(sc);
  // the carried state against C': C_n h_n = C'_n hs_n, hs_n = (n+1) h_n
  float2 hs2[NS / 2];
#pragma unroll
  for (int k = 0; k < NS / 2; ++k) hs2[k] = make_float2((float)(2 * k + 1) * h[2 * k], (float)(2 * k + 2) * h[2 * k + 1]);

  for (int k = w; k < tiles; k += phases) {
    float cum = __ldcg(p.cum + ((int64_t)stream * p.segs_max + k) * kCPW + lane);
    const int64_t t0 = s_begin + (int64_t)k * TILE;
    const int nt = (int)(s_end - t0 < TILE ? s_end - t0 : TILE);
    const int64_t row0 = (int64_t)b * p.len + t0;
    // stage Delta, y and the C rows of the tile
    if (p.fix_vec) {
      constexpr int kRowPieces = kCPW / kChunk;  // 16-byte pieces of a 32-channel row
      for (int i = lane; i < nt * kRowPieces; i += 32) {
        const int r = i / kRowPieces, c = i - r * kRowPieces;
        const bool in = d0 + c * kChunk < p.channels;
        cp_async16_zfill(s_dl + (uint32_t)(r * kCPW + c * kChunk) * sizeof(TIO),
                         in ? (const void*)(dl + (row0 + r) * p.channels + d0 + c * kChunk) : p.delta, in);
      }
      if (y != nullptr)
        for (int i = lane; i < nt * R * kRowPieces; i += 32) {
          const int r = i / kRowPieces, c = i - r * kRowPieces;
          const bool in = d0 + c * kChunk < p.channels;
          cp_async16_zfill(s_y + (uint32_t)(r * kCPW + c * kChunk) * sizeof(TIO),
                           in ? (const void*)(y + (row0 * R + r) * p.channels + d0 + c * kChunk) : p.delta, in);
        }
      constexpr int kCPieces = NS / 4;  // 16-byte pieces of an fp32 C' row
      for (int i = lane; i < nt * R * kCPieces; i += 32)
        cp_async16_zfill(s_c + (uint32_t)i * 16u, Cs + row0 * R * NS + (int64_t)i * 4, true);
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
      for (int r = 0; r < nt; ++r) sdl[r * kCPW + lane] = active ? dl[(row0 + r) * p.channels + d] : from_f32<TIO>(0.0f);
      if (y != nullptr)
        for (int r = 0; r < nt * R; ++r)
          sy[r * kCPW + lane] = active ? y[(row0 * R + r) * p.channels + d] : from_f32<TIO>(0.0f);
      for (int i = lane; i < nt * R * NS; i += 32) sc[i] = Cs[row0 * R * NS + i];
    }
    __syncwarp();
    for (int r = 0; r < nt; ++r) {
      if constexpr (CKPT) {
        if (r == 0 && active) {  // tiles start at multiples of TILE
          float* ck = p.ckpt + (((int64_t)b * ((p.len + TILE - 1) / TILE) + t0 / TILE) * p.channels + d) * NS;
#pragma unroll
          for (int k2 = 0; k2 < NS; ++k2) ck[k2] = fmaf(ex2_approx(cum * an[k2] * kLog2e), h[k2], ck[k2]);
        }
      }
      cum += to_f32(sdl[r * kCPW + lane]);
      // the carried state's decay to this token, exp(A_n cum)
      const float rho = ex2_approx(cum * a0l);
      float ev[NS];
      if (!structured) {
#pragma unroll
        for (int n = 0; n < NS; ++n) ev[n] = ex2_approx(cum * an[n] * kLog2e);
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {  // output q reads the state with its own C row
        // the products C'_n hs_n in pairs (n, n+1)
        float2 pc[NS / 2];
        const float4* crow = reinterpret_cast<const float4*>(sc + (r * R + q) * NS);
#pragma unroll
        for (int i = 0; i < NS / 4; ++i) {
          const float4 v = crow[i];
          pc[2 * i] = __fmul2_rn(make_float2(v.x, v.y), hs2[2 * i]);
          pc[2 * i + 1] = __fmul2_rn(make_float2(v.z, v.w), hs2[2 * i + 1]);
        }
        float corr;
        if (structured) {
          // sum_n C_n h_n rho^(n+1) = rho (E(rho^2) + rho O(rho^2)), E and O
          // the polynomials of the even and the odd states, Horner together
          const float rho2 = rho * rho;
          const float2 rr = make_float2(rho2, rho2);
          float2 acc = pc[NS / 2 - 1];
#pragma unroll
          for (int k = NS / 2 - 2; k >= 0; --k) acc = __ffma2_rn(acc, rr, pc[k]);
          corr = fmaf(acc.y, rho, acc.x) * rho;
        } else {
          corr = 0.0f;
#pragma unroll
          for (int k = 0; k < NS / 2; ++k) corr = fmaf(ev[2 * k], pc[k].x, fmaf(ev[2 * k + 1], pc[k].y, corr));
        }
        TIO& yv = sy[(r * R + q) * kCPW + lane];
        yv = from_f32<TIO>(to_f32(yv) + corr);
      }
    }
    __syncwarp();
    // write y back
    if (y != nullptr) {
      if (p.fix_vec) {
        constexpr int kRowPieces = kCPW / kChunk;
        for (int i = lane; i < nt * R * kRowPieces; i += 32) {
          const int r = i / kRowPieces, c = i - r * kRowPieces;
          if (d0 + c * kChunk < p.channels)
            *reinterpret_cast<uint4*>(y + (row0 * R + r) * p.channels + d0 + c * kChunk) =
                *reinterpret_cast<const uint4*>(sy + r * kCPW + c * kChunk);
        }
      } else if (active) {
        for (int r = 0; r < nt * R; ++r) y[(row0 * R + r) * p.channels + d] = sy[r * kCPW + lane];
      }
    }
    __syncwarp();
    if (__all_sync(0xffffffffu, !active || cum * kmax < -fix_stop_log2<TIO>()))
      break;  // later tiles of this warp add less (their cum is larger)
  }
}

// ---------------------------------------------------------------------------
// pre-pass, one thread per element of three ranges:
//   [0, zero_words):          the job counters and progress flags = 0
//   C' = C / (n+1) in fp32 for every (token row, state), and B widened to
//   fp32 when bs is given (bf16 data): four consecutive states per thread
//   per channel {A[d,0], 1/A[d,0], D[d], structured}, where "structured"
//   means A[d,n] == (n+1) A[d,0] exactly for every n, A[d,0] < 0 and the
//   general path was not forced; padding channels get {-1, -1, 0, 1}.
// ---------------------------------------------------------------------------
template <typename TIO, int NS>
__global__ void scan_prep_kernel(int* __restrict__ zero, int64_t zero_words, const TIO* __restrict__ C,
                                 float* __restrict__ cs, const TIO* __restrict__ B, float* __restrict__ bs,
                                 int64_t total_c, const float* __restrict__ A,
                                 const float* __restrict__ D, float4* __restrict__ chan, int64_t channels,
                                 int64_t chan_padded, int force_general) {
  griddep_launch_dependents();  // the scan kernel may start its setup
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  griddep_wait();  // the scratch may still be in use by the previous kernel of the stream
  if (i < zero_words) {
    zero[i] = 0;
    return;
  }
  i -= zero_words;
  const int64_t quads = total_c / 4;  // four consecutive elements of a row per thread (NS % 4 == 0)
  if (i < quads) {
    const int64_t e = 4 * i;
    const int n = (int)(e % NS);
    reinterpret_cast<float4*>(cs)[i] =
        make_float4(to_f32(C[e]) / (float)(n + 1), to_f32(C[e + 1]) / (float)(n + 2),
                    to_f32(C[e + 2]) / (float)(n + 3), to_f32(C[e + 3]) / (float)(n + 4));
    if (bs)
      reinterpret_cast<float4*>(bs)[i] = make_float4(to_f32(B[e]), to_f32(B[e + 1]), to_f32(B[e + 2]), to_f32(B[e + 3]));
    return;
  }
  const int64_t d = i - quads;
  if (d >= chan_padded) return;
  if (d >= channels) {
    chan[d] = make_float4(-1.0f, -1.0f, 0.0f, 1.0f);
    return;
  }
  const float* row = A + d * NS;
  const float a0 = row[0];
  bool structured = !force_general && a0 < 0.0f;
#pragma unroll
  for (int n = 1; n < NS; ++n) structured &= (row[n] == (float)(n + 1) * a0);
  chan[d] = make_float4(a0, 1.0f / a0, D ? D[d] : 0.0f, structured ? 1.0f : 0.0f);
}

}  // namespace mamba
