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
//   * A "group" is 32 consecutive channels of one batch row; one warp owns a
//     group and each lane owns one channel with its N states in registers.
//   * The sequence of a group is cut into chunks.  A job is (stream, chunk):
//     a warp runs the recurrence over the chunk's tokens starting from the
//     state the previous chunk of the same stream ended with.  Jobs are
//     handed out by an atomic ticket in chunk-major order, so the predecessor
//     of every job was taken earlier by a running warp: waits always end.
//     The grid is persistent (one warp per SM sub-partition), which keeps
//     every sub-partition busy whatever the group count.
//   * When there are fewer groups than warps, the sequence is also cut into
//     "super-chunks" that run as independent streams.  Their starting states
//     come from the associative combine of the page's parallel prefix scan
//     ("Paralel Tarama Algoritması"): an aggregate pass computes, per
//     super-chunk, the end state from zero H_j and sum of Delta; a combine
//     pass runs h_{j+1} = exp(A sum Delta_j) h_j + H_j; the main pass then
//     runs every super-chunk from its own starting state.
//
// Arithmetic per token and state (all fp32; the state is kept scaled,
// g_n = A_n h_n, so that 1/A_n leaves the inner loop):
//     e_n  = expm1(Delta A_n)
//     g_n <- g_n + e_n (g_n + B_n x)          (== Abar g + e B x)
//     y   += (C_n / A_n) g_n
// When A[d,n] == (n+1) A[d,0] for every n of every channel in the warp (the
// S4D-real structure), e_n comes from one exact-arithmetic identity,
//     e^{(n+1) z} - 1 = e^z (e^{n z} - 1) + (e^z - 1),
// i.e. e_n = r e_{n-1} + q with q = expm1(Delta A[d,0]), r = 1 + q: one FMA per
// state instead of an exponential; then C_n / A_n = (C_n / (n+1)) / A_0.
// Otherwise every e_n is computed from its own exponential.
//
// Data path of a tile: u, Delta and B in the I/O type, and C' = C / (n+1) as
// fp32 (one small pre-pass per call), staged by TMA.  With bf16 data the
// input term B_n x is one mixed-precision FMA on the raw bf16 operands
// (their product is exact in fp32); nothing is converted in shared memory.
// Each lane reads the whole B and C' row of every token, so the bytes
// broadcast from shared memory per token are the other limit next to the
// FMA pipe: 32 B of B and 64 B of C' at N = 16.
#pragma once

#include "common.cuh"

namespace mamba {

constexpr int kWarpsPerCta = 4;   // one warp per SM sub-partition
constexpr int kGroup = 32;        // channels per warp
constexpr int kMaxRing = 8;       // jobs a warp may have pulled ahead of its compute

enum ScanMode : int { kModeFull = 0, kModeAggregate = 1 };

struct ScanParams {
  // tensors
  const void* u;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;
  const float* cs;          // C' = C / (n+1), fp32 [batch*len][N] (scratch, written by the pre-pass)
  const float* D;           // nullable
  const float* h0;          // nullable: initial state [b][d][n]
  void* y;
  float* final_state;       // nullable
  // scratch (stream-ordered, zeroed where noted)
  int* counters;            // [0] job ticket, [1] abort flag (zeroed)
  int* done;                // [streams] chunks completed per stream (zeroed)
  float* ring;              // [streams][2][32][N] states handed between chunks
  float* ring_sd;           // [streams][2][32] running sum of Delta (aggregate mode)
  float* agg_h;             // [(S-1)*G][32][N] aggregate end states
  float* agg_sd;            // [(S-1)*G][32]    aggregate sum of Delta
  const float* hin;         // [S*G][32][N] starting state of each super-chunk (S > 1)
  // sizes
  int64_t batch, len, channels;
  int groups_d;             // ceil(channels / 32)
  int groups;               // batch * groups_d
  int supers;               // S
  int64_t super_len;        // tokens per super-chunk (all but the last)
  int64_t chunk_len;        // tokens per chunk
  int chunks_full;          // chunks of a full super-chunk
  int chunks_last;          // chunks of the last super-chunk (full mode)
  int mode;
  int streams;              // streams active in this pass
  int jobs;                 // jobs in this pass (fits int32, checked on the host)
  int use_tma;
  int force_general;
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

__device__ __forceinline__ Job decode_job(const ScanParams& p, int j_in, int tile) {
  // 32-bit arithmetic: the host guarantees jobs, streams and b*len fit in int32
  Job jb;
  const uint32_t j = (uint32_t)j_in;
  const uint32_t n_all = (uint32_t)p.streams;
  const uint32_t n_full = (p.mode == kModeFull) ? (uint32_t)(p.supers - 1) * (uint32_t)p.groups : n_all;
  const uint32_t kmin = (uint32_t)((p.mode == kModeFull) ? p.chunks_last : p.chunks_full);
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
  jb.d0 = (grp - jb.b * p.groups_d) * kGroup;
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
// shared-memory layout of one warp: STAGES tile slots (TMA destinations,
// 128-byte aligned), their full barriers, the warp's job queue
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int TILE, int STAGES>
struct alignas(128) WarpSmem {
  TIO u[STAGES][TILE][kGroup];
  TIO dl[STAGES][TILE][kGroup];
  TIO b[STAGES][TILE][NS];
  float cs[STAGES][TILE][NS];
  uint64_t full[STAGES];
  int ring_jobs[kMaxRing];
};

template <typename TIO, int NS, int TILE, int STAGES>
constexpr size_t scan_smem_bytes() {
  return sizeof(WarpSmem<TIO, NS, TILE, STAGES>) * kWarpsPerCta + 128;
}

template <typename TIO, int NS>
__host__ __device__ constexpr uint32_t tile_bytes(int tile) {
  return (uint32_t)(tile * (2 * kGroup * sizeof(TIO) + NS * sizeof(TIO) + NS * sizeof(float)));
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

// exp(z) - 1 from the hardware exp2 (no branch): absolute error about 1e-7,
// i.e. a relative error below 1e-4 once |z| > 1e-3.  Used for bf16 data.
__device__ __forceinline__ float expm1_fast(float z) { return ex2_approx(z * 1.4426950408889634f) - 1.0f; }

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// d = lo16(w) * x + c and d = hi16(w) * x + c with bf16 multiplicands and an
// fp32 addend (the bf16 x bf16 product is exact in fp32).
__device__ __forceinline__ float fma_bf16_lo(uint32_t w, uint16_t x, float c) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, l, %2, %3;\n\t}"
      : "=f"(d) : "r"(w), "h"(x), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t w, uint16_t x, float c) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, h, %2, %3;\n\t}"
      : "=f"(d) : "r"(w), "h"(x), "f"(c));
  return d;
}

// e2[k] = (exp((2k+1) z) - 1, exp((2k+2) z) - 1) for k < NS/2 from
// q = exp(z) - 1, using exp((m+k) z) - 1 = (exp(k z) - 1) + exp(k z)(exp(m z) - 1):
// the first four by steps of z, the rest by steps of 4z in four independent
// chains (dependency depth 7 instead of NS - 1).
template <int NS>
__device__ __forceinline__ void decay_chain2(float q, float2 (&e2)[NS / 2]) {
  static_assert(NS % 4 == 0, "NS multiple of 4");
  const float r1 = 1.0f + q;
  const float e1 = fmaf(r1, q, q);
  const float e2s = fmaf(r1, e1, q);
  const float e3 = fmaf(r1, e2s, q);
  e2[0] = f2(q, e1);
  e2[1] = f2(e2s, e3);
  const float2 r4 = f2(1.0f + e3, 1.0f + e3);
  const float2 q4 = f2(e3, e3);
#pragma unroll
  for (int k = 2; k < NS / 2; ++k) e2[k] = __ffma2_rn(r4, e2[k - 2], q4);
}

__device__ __forceinline__ uint16_t raw16(__nv_bfloat16 v) { return __bfloat16_as_ushort(v); }

// One token for one lane: g <- g + e (g + B x) for all states; returns
// sum_n C'_n g_n.  States as N/2 float2 pairs, every state step a packed
// FFMA2 except the bf16 input term (two mixed FMAs per pair).
template <typename TIO, int NS>
__device__ __forceinline__ float token_update(const float2 (&e)[NS / 2], const TIO* brow, const float* csrow, TIO xr,
                                              float2 (&g)[NS / 2]) {
  float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
  if constexpr (sizeof(TIO) == 2) {
    const uint16_t xh = raw16(xr);
    uint32_t bw[NS / 2];
#pragma unroll
    for (int k8 = 0; k8 < NS / 8; ++k8) {
      const uint4 w = reinterpret_cast<const uint4*>(brow)[k8];
      bw[4 * k8] = w.x; bw[4 * k8 + 1] = w.y; bw[4 * k8 + 2] = w.z; bw[4 * k8 + 3] = w.w;
    }
#pragma unroll
    for (int n4 = 0; n4 < NS / 4; ++n4) {
      const float4 cv = reinterpret_cast<const float4*>(csrow)[n4];
      const int p0 = 2 * n4, p1 = 2 * n4 + 1;
      const float2 v0 = f2(fma_bf16_lo(bw[p0], xh, g[p0].x), fma_bf16_hi(bw[p0], xh, g[p0].y));
      const float2 v1 = f2(fma_bf16_lo(bw[p1], xh, g[p1].x), fma_bf16_hi(bw[p1], xh, g[p1].y));
      g[p0] = __ffma2_rn(e[p0], v0, g[p0]);
      g[p1] = __ffma2_rn(e[p1], v1, g[p1]);
      acc0 = __ffma2_rn(f2(cv.x, cv.y), g[p0], acc0);
      acc1 = __ffma2_rn(f2(cv.z, cv.w), g[p1], acc1);
    }
  } else {
    const float x = to_f32(xr);
    const float2 x2 = f2(x, x);
#pragma unroll
    for (int n4 = 0; n4 < NS / 4; ++n4) {
      const float4 bv = reinterpret_cast<const float4*>(brow)[n4];
      const float4 cv = reinterpret_cast<const float4*>(csrow)[n4];
      const int p0 = 2 * n4, p1 = 2 * n4 + 1;
      const float2 v0 = __ffma2_rn(f2(bv.x, bv.y), x2, g[p0]);
      const float2 v1 = __ffma2_rn(f2(bv.z, bv.w), x2, g[p1]);
      g[p0] = __ffma2_rn(e[p0], v0, g[p0]);
      g[p1] = __ffma2_rn(e[p1], v1, g[p1]);
      acc0 = __ffma2_rn(f2(cv.x, cv.y), g[p0], acc0);
      acc1 = __ffma2_rn(f2(cv.z, cv.w), g[p1], acc1);
    }
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// Rows [0, rows) of one tile, structured A.  FULL: write y; otherwise
// accumulate sum(Delta).  FASTQ: expm1(Delta A_0) from the hardware exp2.
// Two tokens per step: their decay chains are independent work for the
// scheduler while the state updates wait on each other.
template <typename TIO, int NS, int TILE, bool FULL, bool FASTQ>
__device__ __forceinline__ void tile_structured(const TIO* su, const TIO* sdl, const TIO (*bt)[NS],
                                                const float (*ct)[NS], int rows, float a0, float inv_a0, float Dd,
                                                float2 (&g)[NS / 2], float& sd, TIO* yp, int64_t ystride,
                                                bool active) {
  const float a0l2e = a0 * 1.4426950408889634f;
  auto chain = [&](float dt, float2 (&e)[NS / 2]) {
    const float q = FASTQ ? ex2_approx(dt * a0l2e) - 1.0f : expm1_small(dt * a0);
    decay_chain2<NS>(q, e);
  };
  auto emit = [&](float s, TIO xr, float dt) {
    if constexpr (FULL) {
      if (active) *yp = from_f32<TIO>(fmaf(s, inv_a0, Dd * to_f32(xr)));
      yp += ystride;
    } else {
      sd += dt;
    }
  };
  auto pair = [&](int r) {
    const TIO x0 = su[r * kGroup], x1 = su[(r + 1) * kGroup];
    const float d0 = to_f32(sdl[r * kGroup]), d1 = to_f32(sdl[(r + 1) * kGroup]);
    float2 e0[NS / 2], e1[NS / 2];
    chain(d0, e0);
    chain(d1, e1);
    const float s0 = token_update<TIO, NS>(e0, bt[r], ct[r], x0, g);
    const float s1 = token_update<TIO, NS>(e1, bt[r + 1], ct[r + 1], x1, g);
    emit(s0, x0, d0);
    emit(s1, x1, d1);
  };
  int r = 0;
  if (rows == TILE) {
#pragma unroll 4
    for (; r < TILE; r += 2) pair(r);
  } else {
    for (; r + 1 < rows; r += 2) pair(r);
    if (r < rows) {
      const TIO x0 = su[r * kGroup];
      const float d0 = to_f32(sdl[r * kGroup]);
      float2 e0[NS / 2];
      chain(d0, e0);
      emit(token_update<TIO, NS>(e0, bt[r], ct[r], x0, g), x0, d0);
    }
  }
}

// Rows [0, rows) of one tile, general A: one exponential per state.
// kA[n] = A_n log2(e), kC[n] = (n+1) / A_n (so that C'_n kC[n] = C_n / A_n).
template <typename TIO, int NS, bool FULL>
__device__ __forceinline__ void tile_general(const TIO* su, const TIO* sdl, const TIO (*bt)[NS],
                                             const float (*ct)[NS], int rows, const float (&kA)[NS],
                                             const float (&kC)[NS], float Dd, float2 (&g)[NS / 2], float& sd,
                                             TIO* yp, int64_t ystride, bool active) {
  for (int r = 0; r < rows; ++r) {
    const TIO xr = su[r * kGroup];
    const float dt = to_f32(sdl[r * kGroup]);
    float2 e[NS / 2];
#pragma unroll
    for (int k = 0; k < NS / 2; ++k) {
      float e0, e1;
      if constexpr (sizeof(TIO) == 4) {  // fp32 data: accurate expm1
        e0 = expm1_small(dt * (kA[2 * k] * 0.69314718055994531f));
        e1 = expm1_small(dt * (kA[2 * k + 1] * 0.69314718055994531f));
      } else {
        e0 = ex2_approx(dt * kA[2 * k]) - 1.0f;
        e1 = ex2_approx(dt * kA[2 * k + 1]) - 1.0f;
      }
      e[k] = f2(e0, e1);
    }
    float crow[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) crow[n] = ct[r][n] * kC[n];
    const float s = token_update<TIO, NS>(e, bt[r], crow, xr, g);
    if constexpr (FULL) {
      if (active) *yp = from_f32<TIO>(s + Dd * to_f32(xr));
      yp += ystride;
    } else {
      sd += dt;
    }
  }
}

// ---------------------------------------------------------------------------
// per-warp context: tile pipeline (producer in lane 0) and job queue
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int TILE, int STAGES>
struct WarpCtx {
  using Smem = WarpSmem<TIO, NS, TILE, STAGES>;
  const ScanParams& p;
  Smem& sm;
  const CUtensorMap* mu;
  const CUtensorMap* mdl;
  const CUtensorMap* mb;
  const CUtensorMap* mc;
  int lane;
  // producer (meaningful in lane 0): ring index of the job being loaded,
  // its next tile, jobs pulled so far; tiles issued / consumed
  uint32_t ld_ring = 0, pulled = 0, cm_ring = 0;
  int ld_tile = 0, ld_ntiles = 0, ld_row0 = 0, ld_d0 = 0;
  bool ld_done = false;
  uint32_t ld_seq = 0, cm_seq = 0;

  __device__ WarpCtx(const ScanParams& p_, Smem& sm_, const CUtensorMap* a, const CUtensorMap* b,
                     const CUtensorMap* c, const CUtensorMap* d, int lane_)
      : p(p_), sm(sm_), mu(a), mdl(b), mb(c), mc(d), lane(lane_) {}

  __device__ int pull_job() {  // lane 0
    int j = atomicAdd(&p.counters[0], 1);
    if (j >= p.jobs || ld_volatile(&p.counters[1]) != 0) j = -1;
    sm.ring_jobs[pulled % kMaxRing] = j;
    ++pulled;
    return j;
  }

  // issue loads until STAGES tiles are ahead of the compute side (lane 0)
  __device__ void produce() {
    while (!ld_done && ld_seq < cm_seq + STAGES) {
      if (ld_tile >= ld_ntiles) {
        if (ld_ring + 1 >= pulled) {
          if (pulled - cm_ring >= (uint32_t)kMaxRing) break;  // queue full
          if (pull_job() < 0) { ld_done = true; break; }
        }
        ++ld_ring;
        const int j = sm.ring_jobs[ld_ring % kMaxRing];
        if (j < 0) { ld_done = true; break; }
        const Job jb = decode_job(p, j, TILE);
        ld_tile = 0;
        ld_ntiles = jb.ntiles;
        ld_row0 = (int)(jb.b * p.len + jb.t0);
        ld_d0 = jb.d0;
        continue;
      }
      const int slot = ld_seq % STAGES;
      const int row = ld_row0 + ld_tile * TILE;
      if (p.use_tma) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&sm.full[slot], tile_bytes<TIO, NS>(TILE));
        tma_load_2d(&sm.u[slot][0][0], mu, &sm.full[slot], ld_d0, row);
        tma_load_2d(&sm.dl[slot][0][0], mdl, &sm.full[slot], ld_d0, row);
        tma_load_2d(&sm.b[slot][0][0], mb, &sm.full[slot], 0, row);
        tma_load_2d(&sm.cs[slot][0][0], mc, &sm.full[slot], 0, row);
      } else {
        mbar_arrive(&sm.full[slot]);  // the warp fetches the tile itself at consume time
      }
      ++ld_tile;
      ++ld_seq;
    }
  }

  // next job id for the compute side (all lanes), -1 when done
  __device__ int next_job() {
    ++cm_ring;
    int jsel = -1;
    if (lane == 0) {
      produce();
      while (!ld_done && cm_ring >= pulled) {
        if (pull_job() < 0) ld_done = true;
      }
      jsel = (cm_ring < pulled) ? sm.ring_jobs[cm_ring % kMaxRing] : -1;
    }
    return __shfl_sync(0xffffffffu, jsel, 0);
  }

  __device__ void abort_all() {  // lane 0
    record_device_error(MAMBA_ERR_TIMEOUT);
    atomicExch(&p.counters[1], 1);
  }

  // wait until the previous chunk of the stream has handed its state on
  __device__ bool wait_predecessor(const Job& jb) {
    bool aborted = false;
    if (lane == 0) {
      const uint64_t t_start = globaltimer_ns();
      uint32_t spins = 0;
      while (ld_acquire(&p.done[jb.stream]) < jb.chunk) {
        if (ld_volatile(&p.counters[1]) != 0) { aborted = true; break; }
        if ((++spins & 31u) == 0 && globaltimer_ns() - t_start > p.wait_limit_ns) {
          abort_all();
          aborted = true;
          break;
        }
        __nanosleep(spins < 64 ? 32 : 256);
      }
    }
    aborted = __shfl_sync(0xffffffffu, (int)aborted, 0) != 0;
    if (!aborted) (void)ld_acquire(&p.done[jb.stream]);  // every lane acquires before reading the state
    return !aborted;
  }

  // wait for the next tile; the plain-load path fetches it here
  __device__ bool acquire_tile(const Job& jb, int64_t tt0, int rows, int d, bool active) {
    const int slot = cm_seq % STAGES;
    bool ok = mbar_wait_bounded(&sm.full[slot], (cm_seq / STAGES) & 1u, p.wait_limit_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) abort_all();
      return false;
    }
    if (!p.use_tma) {
      const TIO* gu = static_cast<const TIO*>(p.u);
      const TIO* gdl = static_cast<const TIO*>(p.delta);
      const TIO* gB = static_cast<const TIO*>(p.B);
      const int64_t rowbase = (int64_t)jb.b * p.len + tt0;
      for (int r = 0; r < rows; ++r) {
        const int64_t off = (rowbase + r) * p.channels + d;
        sm.u[slot][r][lane] = active ? gu[off] : from_f32<TIO>(0.0f);
        sm.dl[slot][r][lane] = active ? gdl[off] : from_f32<TIO>(0.0f);
      }
      for (int i = lane; i < rows * NS; i += 32) {
        const int r = i / NS, n = i - r * NS;
        sm.b[slot][r][n] = gB[(rowbase + r) * NS + n];
        sm.cs[slot][r][n] = p.cs[(rowbase + r) * NS + n];
      }
      __syncwarp();
    }
    return true;
  }

  // the tile is consumed: refill its slot
  __device__ void release_tile() {
    __syncwarp();
    ++cm_seq;
    if (lane == 0) produce();
    __syncwarp();
  }
};

// One job: the recurrence over the chunk's tokens for the warp's 32 channels,
// from the state the previous chunk handed on, then hand the end state on.
// STRUCT: A[d,n] = (n+1) A[d,0] on every lane (see decay_chain2).
template <typename TIO, int NS, int TILE, int STAGES, bool STRUCT, bool FULL>
__device__ __forceinline__ bool run_job(WarpCtx<TIO, NS, TILE, STAGES>& cx, const Job& jb, float a0) {
  const ScanParams& p = cx.p;
  auto& sm = cx.sm;
  const int lane = cx.lane;
  const int d = jb.d0 + lane;
  const bool active = d < p.channels;
  const float Dd = (FULL && active && p.D) ? __ldg(p.D + d) : 0.0f;
  const float* Arow = p.A + (int64_t)(active ? d : 0) * NS;

  if (!jb.first && !cx.wait_predecessor(jb)) return false;

  // starting state, kept scaled: g_n = A_n h_n
  float2 g[NS / 2];
  float sd = 0.0f;
  {
    const float* src = nullptr;
    if (!jb.first) {
      const int64_t slot_i = (int64_t)jb.stream * 2 + ((jb.chunk - 1) & 1);
      src = p.ring + slot_i * (kGroup * NS) + lane * NS;
      if (!FULL) sd = p.ring_sd[slot_i * kGroup + lane];
    } else if (FULL) {
      if (jb.super_idx > 0) src = p.hin + ((int64_t)jb.stream * kGroup + lane) * NS;
      else if (p.h0 && active) src = p.h0 + ((int64_t)jb.b * p.channels + d) * NS;
    }
#pragma unroll
    for (int k = 0; k < NS / 2; ++k) {
      float ak0, ak1;
      if constexpr (STRUCT) {
        ak0 = (float)(2 * k + 1) * a0;
        ak1 = (float)(2 * k + 2) * a0;
      } else {
        ak0 = active ? __ldg(Arow + 2 * k) : -1.0f;
        ak1 = active ? __ldg(Arow + 2 * k + 1) : -1.0f;
      }
      g[k] = src ? f2(src[2 * k] * ak0, src[2 * k + 1] * ak1) : f2(0.0f, 0.0f);
    }
  }

  TIO* yrow = static_cast<TIO*>(p.y) + ((int64_t)jb.b * p.len + jb.t0) * p.channels + d;
  for (int it = 0; it < jb.ntiles; ++it) {
    const int64_t tt0 = jb.t0 + (int64_t)it * TILE;
    const int rows = (int)(jb.t1 - tt0 < (int64_t)TILE ? jb.t1 - tt0 : (int64_t)TILE);
    if (!cx.acquire_tile(jb, tt0, rows, d, active)) return false;
    const int slot = cx.cm_seq % STAGES;
    const TIO* su = &sm.u[slot][0][lane];
    const TIO* sdl = &sm.dl[slot][0][lane];
    if constexpr (STRUCT) {
      constexpr bool kFastQ = sizeof(TIO) == 2;  // bf16 data: hardware exp2 for expm1(Delta A_0)
      tile_structured<TIO, NS, TILE, FULL, kFastQ>(su, sdl, sm.b[slot], sm.cs[slot], rows, a0, 1.0f / a0, Dd, g,
                                                   sd, yrow, p.channels, active);
    } else {
      float kA[NS], kC[NS];
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        const float an = active ? __ldg(Arow + n) : -1.0f;
        kA[n] = an * 1.4426950408889634f;
        kC[n] = (float)(n + 1) / an;
      }
      tile_general<TIO, NS, FULL>(su, sdl, sm.b[slot], sm.cs[slot], rows, kA, kC, Dd, g, sd, yrow, p.channels,
                                  active);
    }
    yrow += (int64_t)rows * p.channels;
    cx.release_tile();
  }

  // hand the end state on (unscaled)
  float* dst;
  float* dst_sd = nullptr;
  if (!jb.last) {
    const int64_t slot_i = (int64_t)jb.stream * 2 + (jb.chunk & 1);
    dst = p.ring + slot_i * (kGroup * NS) + lane * NS;
    if (!FULL) dst_sd = p.ring_sd + slot_i * kGroup + lane;
  } else if (FULL) {
    dst = (p.final_state && active && jb.super_idx == p.supers - 1)
              ? p.final_state + ((int64_t)jb.b * p.channels + d) * NS
              : nullptr;
  } else {
    dst = p.agg_h + ((int64_t)jb.stream * kGroup + lane) * NS;
    dst_sd = p.agg_sd + (int64_t)jb.stream * kGroup + lane;
  }
  if (dst) {
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      float inv;
      if constexpr (STRUCT) inv = 1.0f / ((float)(n + 1) * a0);
      else inv = active ? 1.0f / __ldg(Arow + n) : -1.0f;
      dst[n] = ((n & 1) ? g[n >> 1].y : g[n >> 1].x) * inv;
    }
  }
  if (dst_sd) *dst_sd = sd;
  if (!jb.last) {
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release(&p.done[jb.stream], jb.chunk + 1);
  }
  __syncwarp();
  return true;
}

// ---------------------------------------------------------------------------
// the persistent chunked scan kernel
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int TILE, int STAGES>
__global__ void __launch_bounds__(kWarpsPerCta * 32, 1)
scan_chunks_kernel(const __grid_constant__ ScanParams p, const __grid_constant__ CUtensorMap map_u,
                   const __grid_constant__ CUtensorMap map_dl, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_c) {
  using Smem = WarpSmem<TIO, NS, TILE, STAGES>;
  // TMA destinations must start on 128-byte boundaries
  static_assert(sizeof(Smem) % 128 == 0, "per-warp block keeps 128-byte alignment");
  static_assert((sizeof(TIO) * TILE * kGroup) % 128 == 0 && (sizeof(TIO) * TILE * NS) % 128 == 0,
                "tile slots keep 128-byte alignment");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // align to 128 bytes by pointer arithmetic (an integer round trip would
  // hide from the compiler that these are shared-memory addresses)
  unsigned char* smem_base = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  Smem& sm = reinterpret_cast<Smem*>(smem_base)[warp];

  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    fence_mbar_init();
    if (p.use_tma) {
      tma_prefetch_desc(&map_u);
      tma_prefetch_desc(&map_dl);
      tma_prefetch_desc(&map_b);
      tma_prefetch_desc(&map_c);
    }
  }
  __syncwarp();

  WarpCtx<TIO, NS, TILE, STAGES> cx(p, sm, &map_u, &map_dl, &map_b, &map_c, lane);
  // ring entry 0 is a sentinel "before the first job": the first produce()
  // pulls job #1 into entry 1
  if (lane == 0) {
    sm.ring_jobs[0] = -1;
    cx.pulled = 1;
    cx.produce();
  }
  __syncwarp();

  const bool full_mode = (p.mode == kModeFull);
  for (;;) {
    const int j = cx.next_job();
    if (j < 0) break;
    const Job jb = decode_job(p, j, TILE);
    const int d = jb.d0 + lane;
    const bool active = d < p.channels;
    // structured A: A[d,n] == (n+1) A[d,0] exactly, on every lane of the warp
    const float* Arow = p.A + (int64_t)(active ? d : 0) * NS;
    const float a0 = active ? __ldg(Arow) : -1.0f;
    bool structured = !p.force_general && a0 < 0.0f;
#pragma unroll
    for (int n = 1; n < NS; ++n) structured = structured && (!active || __ldg(Arow + n) == (float)(n + 1) * a0);
    structured = __all_sync(0xffffffffu, structured);
    bool ok;
    if (structured)
      ok = full_mode ? run_job<TIO, NS, TILE, STAGES, true, true>(cx, jb, a0)
                     : run_job<TIO, NS, TILE, STAGES, true, false>(cx, jb, a0);
    else
      ok = full_mode ? run_job<TIO, NS, TILE, STAGES, false, true>(cx, jb, a0)
                     : run_job<TIO, NS, TILE, STAGES, false, false>(cx, jb, a0);
    if (!ok) break;
  }

  // Drain: every TMA load this warp issued must land before the CTA exits.
  __syncwarp();
  if (lane == 0 && p.use_tma) {
    for (uint32_t s = cx.cm_seq; s < cx.ld_seq; ++s) {
      if (!mbar_wait_bounded(&sm.full[s % STAGES], (s / STAGES) & 1u, p.wait_limit_ns)) {
        record_device_error(MAMBA_ERR_TIMEOUT);
        break;
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// pre-pass: C' = C / (n+1) in fp32, one thread per (token row, state)
// ---------------------------------------------------------------------------
template <typename TIO, int NS>
__global__ void scan_prep_c_kernel(const TIO* __restrict__ C, float* __restrict__ cs, int64_t total) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int n = (int)(i % NS);
  cs[i] = to_f32(C[i]) / (float)(n + 1);
}

// ---------------------------------------------------------------------------
// combine pass: starting state of every super-chunk from the aggregates,
//   h_{j+1} = exp(A * sumDelta_j) h_j + H_j,   h_0 = initial state or 0
// one thread per (group, lane, state).
// ---------------------------------------------------------------------------
template <int NS>
__global__ void scan_combine_kernel(const ScanParams p, float* hin) {
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)p.groups * kGroup * NS;
  if (tid >= total) return;
  const int n = (int)(tid % NS);
  const int lane = (int)((tid / NS) % kGroup);
  const int grp = (int)(tid / ((int64_t)NS * kGroup));
  const int b = grp / p.groups_d;
  const int d = (grp - b * p.groups_d) * kGroup + lane;
  const bool active = d < p.channels;
  const float a = active ? p.A[(int64_t)d * NS + n] : -1.0f;
  float h = (active && p.h0) ? p.h0[((int64_t)b * p.channels + d) * NS + n] : 0.0f;
  for (int j = 0; j + 1 < p.supers; ++j) {
    const int64_t s = (int64_t)j * p.groups + grp;
    const float sdj = p.agg_sd[s * kGroup + lane];
    const float H = p.agg_h[(s * kGroup + lane) * NS + n];
    h = fmaf(expf(a * sdj), h, H);
    hin[(((int64_t)(j + 1) * p.groups + grp) * kGroup + lane) * NS + n] = h;
  }
}

}  // namespace mamba
