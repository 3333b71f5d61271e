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
// state instead of an exponential.  Otherwise every e_n is computed from its
// own exponential.
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
  int64_t chunk_len;        // tokens per chunk (multiple of the tile)
  int chunks_full;          // chunks of a full super-chunk
  int chunks_last;          // chunks of the last super-chunk (full mode)
  int mode;
  int streams;              // streams active in this pass
  int64_t jobs;             // jobs in this pass
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

__device__ __forceinline__ Job decode_job(const ScanParams& p, int64_t j, int tile) {
  Job jb;
  const int64_t n_all = p.streams;                       // streams with >= k+1 chunks for k < kmin
  const int64_t n_full = (p.mode == kModeFull) ? (int64_t)(p.supers - 1) * p.groups : n_all;
  const int kmin = (p.mode == kModeFull) ? p.chunks_last : p.chunks_full;
  int64_t k, s;
  if (j < (int64_t)kmin * n_all) {
    k = j / n_all;
    s = j - k * n_all;
  } else {
    const int64_t jj = j - (int64_t)kmin * n_all;
    k = kmin + jj / n_full;
    s = jj - (k - kmin) * n_full;
  }
  jb.stream = (int)s;
  jb.chunk = (int)k;
  jb.super_idx = (int)(s / p.groups);
  const int grp = (int)(s - (int64_t)jb.super_idx * p.groups);
  jb.b = grp / p.groups_d;
  jb.d0 = (grp - jb.b * p.groups_d) * kGroup;
  const int64_t s_begin = (int64_t)jb.super_idx * p.super_len;
  const int64_t s_end = (s_begin + p.super_len < p.len) ? s_begin + p.super_len : p.len;
  jb.t0 = s_begin + k * p.chunk_len;
  jb.t1 = (jb.t0 + p.chunk_len < s_end) ? jb.t0 + p.chunk_len : s_end;
  jb.ntiles = (int)((jb.t1 - jb.t0 + tile - 1) / tile);
  jb.first = (k == 0);
  jb.last = (jb.t1 == s_end);
  return jb;
}

// ---------------------------------------------------------------------------
// shared-memory layout of one warp
// ---------------------------------------------------------------------------
template <typename TIO, int NS, int TILE, int STAGES>
struct alignas(128) WarpSmem {
  TIO u[STAGES][TILE][kGroup];
  TIO dl[STAGES][TILE][kGroup];
  TIO b[STAGES][TILE][NS];
  TIO c[STAGES][TILE][NS];
  float bf[TILE][NS];   // B as fp32
  float cf[TILE][NS];   // C as fp32 (scaled per path, see below)
  uint64_t full[STAGES];
  int64_t ring_jobs[kMaxRing];
};

template <typename TIO, int NS, int TILE, int STAGES>
constexpr size_t scan_smem_bytes() {
  return sizeof(WarpSmem<TIO, NS, TILE, STAGES>) * kWarpsPerCta + 128;
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
  Smem& sm = reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127))[warp];

  const int64_t L = p.len;
  const int64_t Dch = p.channels;
  const TIO* __restrict__ gu = static_cast<const TIO*>(p.u);
  const TIO* __restrict__ gdl = static_cast<const TIO*>(p.delta);
  const TIO* __restrict__ gB = static_cast<const TIO*>(p.B);
  const TIO* __restrict__ gC = static_cast<const TIO*>(p.C);
  TIO* __restrict__ gy = static_cast<TIO*>(p.y);
  const bool full_mode = (p.mode == kModeFull);

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

  // ---- producer state (meaningful in lane 0; the ring is shared) ----
  int64_t ld_ring = 0;       // ring index of the job being loaded
  int ld_tile = 0;           // next tile of that job to load
  int ld_ntiles = 0;
  int64_t ld_t0 = 0;
  int ld_b = 0, ld_d0 = 0;
  bool ld_done = false;      // no more jobs
  int64_t pulled = 0;        // jobs pulled so far (ring entries)
  uint32_t ld_seq = 0;       // tiles issued
  int64_t cm_ring = 0;       // ring index the compute side is on

  auto pull_job = [&]() -> int64_t {  // lane 0 only
    int64_t j = atomicAdd(&p.counters[0], 1);
    if (j >= p.jobs || ld_volatile(&p.counters[1]) != 0) j = -1;
    sm.ring_jobs[pulled % kMaxRing] = j;
    ++pulled;
    return j;
  };

  // issue loads until STAGES tiles are in flight or nothing is left (lane 0)
  auto produce = [&](uint32_t consumed) {
    while (!ld_done && ld_seq < consumed + STAGES) {
      if (ld_tile >= ld_ntiles) {
        // advance to the next job (pull a new one if needed)
        if (ld_ring + 1 >= pulled) {
          if (pulled - cm_ring >= kMaxRing) break;  // ring full: wait for the compute side
          if (pull_job() < 0) { ld_done = true; break; }
        }
        ++ld_ring;
        const int64_t j = sm.ring_jobs[ld_ring % kMaxRing];
        if (j < 0) { ld_done = true; break; }
        const Job jb = decode_job(p, j, TILE);
        ld_tile = 0;
        ld_ntiles = jb.ntiles;
        ld_t0 = jb.t0;
        ld_b = jb.b;
        ld_d0 = jb.d0;
        continue;
      }
      const int slot = ld_seq % STAGES;
      const int row = (int)(ld_b * L + ld_t0 + (int64_t)ld_tile * TILE);
      if (p.use_tma) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&sm.full[slot], (uint32_t)(sizeof(TIO) * TILE * (2 * kGroup + 2 * NS)));
        tma_load_2d(&sm.u[slot][0][0], &map_u, &sm.full[slot], ld_d0, row);
        tma_load_2d(&sm.dl[slot][0][0], &map_dl, &sm.full[slot], ld_d0, row);
        tma_load_2d(&sm.b[slot][0][0], &map_b, &sm.full[slot], 0, row);
        tma_load_2d(&sm.c[slot][0][0], &map_c, &sm.full[slot], 0, row);
      } else {
        mbar_arrive(&sm.full[slot]);  // data is fetched by the warp at consume time
      }
      ++ld_tile;
      ++ld_seq;
    }
  };

  // ring entry 0 is a sentinel "before the first job": ld_ring starts at 0
  // with ld_ntiles 0, so the first produce() pulls job #1 into entry 1.
  if (lane == 0) {
    sm.ring_jobs[0] = -1;
    pulled = 1;
    produce(0);
  }
  __syncwarp();

  // ---- per-lane constants that depend on the channel are set per job ----
  uint32_t cm_seq = 0;  // tiles consumed
  bool aborted = false;

  for (;;) {
    // next job for the compute side: lane 0 tops up loads (which also pulls
    // jobs) and, if the producer stopped short, pulls the job itself
    ++cm_ring;
    long long jsel = -1;
    if (lane == 0) {
      produce(cm_seq);
      while (!ld_done && cm_ring >= pulled) {
        if (pull_job() < 0) ld_done = true;
      }
      jsel = (cm_ring < pulled) ? (long long)sm.ring_jobs[cm_ring % kMaxRing] : -1;
    }
    const int64_t j = (int64_t)__shfl_sync(0xffffffffu, jsel, 0);
    if (j < 0 || aborted) break;
    const Job jb = decode_job(p, j, TILE);
    const int d = jb.d0 + lane;
    const bool active = d < Dch;

    // ---- per-channel constants ----
    float Arow[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) Arow[n] = active ? __ldg(p.A + (int64_t)d * NS + n) : -(float)(n + 1);
    bool structured = !p.force_general && Arow[0] < 0.0f;
#pragma unroll
    for (int n = 1; n < NS; ++n) structured = structured && (Arow[n] == (float)(n + 1) * Arow[0]);
    structured = __all_sync(0xffffffffu, structured);
    const float a0 = Arow[0];
    const float Dd = (active && p.D) ? __ldg(p.D + d) : 0.0f;

    // ---- starting state ----
    if (!jb.first) {
      if (lane == 0) {
        const uint64_t t_start = globaltimer_ns();
        uint32_t spins = 0;
        while (ld_acquire(&p.done[jb.stream]) < jb.chunk) {
          if (ld_volatile(&p.counters[1]) != 0) { aborted = true; break; }
          if ((++spins & 31u) == 0 && globaltimer_ns() - t_start > p.wait_limit_ns) {
            record_device_error(MAMBA_ERR_TIMEOUT);
            atomicExch(&p.counters[1], 1);
            aborted = true;
            break;
          }
          __nanosleep(64);
        }
      }
      aborted = __shfl_sync(0xffffffffu, (int)aborted, 0) != 0;
      if (aborted) break;
      (void)ld_acquire(&p.done[jb.stream]);  // every lane acquires before reading the state
    }
    float g[NS];   // scaled state g_n = A_n h_n
    float sd = 0.0f;
    {
      const float* src = nullptr;
      if (!jb.first) {
        src = p.ring + ((int64_t)jb.stream * 2 + ((jb.chunk - 1) & 1)) * (kGroup * NS) + lane * NS;
        if (!full_mode) sd = p.ring_sd[((int64_t)jb.stream * 2 + ((jb.chunk - 1) & 1)) * kGroup + lane];
      } else if (full_mode) {
        if (jb.super_idx > 0) src = p.hin + ((int64_t)jb.stream * kGroup + lane) * NS;
        else if (p.h0 && active) src = p.h0 + ((int64_t)jb.b * Dch + d) * NS;
      }
#pragma unroll
      for (int n = 0; n < NS; ++n) g[n] = src ? src[n] * Arow[n] : 0.0f;
    }

    // per-path constants
    float kA[NS];   // structured: unused; general: A_n * log2(e)
    float kC[NS];   // general: 1 / A_n
    float inv_a0 = 1.0f / a0;
    if (!structured) {
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        kA[n] = Arow[n] * 1.4426950408889634f;
        kC[n] = 1.0f / Arow[n];
      }
    }

    // ---- tiles ----
    for (int it = 0; it < jb.ntiles && !aborted; ++it) {
      const int slot = cm_seq % STAGES;
      const uint32_t parity = (cm_seq / STAGES) & 1u;
      const int64_t tt0 = jb.t0 + (int64_t)it * TILE;
      const int rows = (int)(jb.t1 - tt0 < (int64_t)TILE ? jb.t1 - tt0 : (int64_t)TILE);
      bool ok = mbar_wait_bounded(&sm.full[slot], parity, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) {
          record_device_error(MAMBA_ERR_TIMEOUT);
          atomicExch(&p.counters[1], 1);
        }
        aborted = true;
        break;
      }
      if (!p.use_tma) {
        // fetch the tile with plain loads (shapes the TMA path cannot describe)
        const int64_t rowbase = (int64_t)jb.b * L + tt0;
        for (int r = 0; r < rows; ++r) {
          const int64_t off = (rowbase + r) * Dch + d;
          sm.u[slot][r][lane] = active ? gu[off] : from_f32<TIO>(0.0f);
          sm.dl[slot][r][lane] = active ? gdl[off] : from_f32<TIO>(0.0f);
        }
        for (int i = lane; i < rows * NS; i += 32) {
          const int r = i / NS, n = i - r * NS;
          sm.b[slot][r][n] = gB[(rowbase + r) * NS + n];
          sm.c[slot][r][n] = gC[(rowbase + r) * NS + n];
        }
        __syncwarp();
      }
      // B, C -> fp32.  The C operand of the output sum is C_n / A_n: for the
      // structured path 1/A_n = (1/A_0) / (n+1), and 1/(n+1) is folded here
      // (1/A_0 is applied once per output); the general path multiplies by
      // 1/A_n in the loop.
      for (int i = lane; i < rows * NS; i += 32) {
        const int r = i / NS, n = i - r * NS;
        sm.bf[r][n] = to_f32(sm.b[slot][r][n]);
        const float cv = to_f32(sm.c[slot][r][n]);
        sm.cf[r][n] = structured ? cv * (1.0f / (float)(n + 1)) : cv;
      }
      __syncwarp();

      TIO* yrow = gy + ((int64_t)jb.b * L + tt0) * Dch + d;
      if (structured) {
        for (int r = 0; r < rows; ++r) {
          const float x = to_f32(sm.u[slot][r][lane]);
          const float dt = to_f32(sm.dl[slot][r][lane]);
          const float z = dt * a0;
          const float q = expm1_neg(z);
          const float rr = 1.0f + q;
          const float4* b4 = reinterpret_cast<const float4*>(&sm.bf[r][0]);
          const float4* c4 = reinterpret_cast<const float4*>(&sm.cf[r][0]);
          float e = q;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int n4 = 0; n4 < NS / 4; ++n4) {
            const float4 bv = b4[n4];
            const float4 cv = c4[n4];
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
            const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int n = n4 * 4 + k;
              if (n > 0) e = fmaf(rr, e, q);
              const float v = fmaf(bb[k], x, g[n]);
              g[n] = fmaf(e, v, g[n]);
              acc[k] = fmaf(cc[k], g[n], acc[k]);
            }
          }
          sd += dt;
          if (full_mode && active) {
            const float yv = fmaf((acc[0] + acc[1]) + (acc[2] + acc[3]), inv_a0, Dd * x);
            yrow[(int64_t)r * Dch] = from_f32<TIO>(yv);
          }
        }
      } else {
        for (int r = 0; r < rows; ++r) {
          const float x = to_f32(sm.u[slot][r][lane]);
          const float dt = to_f32(sm.dl[slot][r][lane]);
          const float4* b4 = reinterpret_cast<const float4*>(&sm.bf[r][0]);
          const float4* c4 = reinterpret_cast<const float4*>(&sm.cf[r][0]);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int n4 = 0; n4 < NS / 4; ++n4) {
            const float4 bv = b4[n4];
            const float4 cv = c4[n4];
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
            const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int n = n4 * 4 + k;
              float e;
              if constexpr (sizeof(TIO) == 4) {
                e = expm1f(dt * Arow[n]);
              } else {
                e = ex2_approx(dt * kA[n]) - 1.0f;
              }
              const float v = fmaf(bb[k], x, g[n]);
              g[n] = fmaf(e, v, g[n]);
              acc[k] = fmaf(cc[k] * kC[n], g[n], acc[k]);
            }
          }
          sd += dt;
          if (full_mode && active) {
            const float yv = fmaf(1.0f, (acc[0] + acc[1]) + (acc[2] + acc[3]), Dd * x);
            yrow[(int64_t)r * Dch] = from_f32<TIO>(yv);
          }
        }
      }
      __syncwarp();
      ++cm_seq;
      if (lane == 0) produce(cm_seq);
      __syncwarp();
    }
    if (aborted) break;

    // ---- hand the end state on ----
    float* dst;
    float* dst_sd = nullptr;
    if (!jb.last) {
      const int64_t slot_i = (int64_t)jb.stream * 2 + (jb.chunk & 1);
      dst = p.ring + slot_i * (kGroup * NS) + lane * NS;
      if (!full_mode) dst_sd = p.ring_sd + slot_i * kGroup + lane;
    } else if (full_mode) {
      dst = (p.final_state && active && jb.super_idx == p.supers - 1)
                ? p.final_state + ((int64_t)jb.b * Dch + d) * NS
                : nullptr;
    } else {
      dst = p.agg_h + ((int64_t)jb.stream * kGroup + lane) * NS;
      dst_sd = p.agg_sd + (int64_t)jb.stream * kGroup + lane;
    }
    if (dst) {
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        const float inv = structured ? inv_a0 * (1.0f / (float)(n + 1)) : kC[n];
        dst[n] = g[n] * inv;
      }
    }
    if (dst_sd) *dst_sd = sd;
    if (!jb.last) {
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release(&p.done[jb.stream], jb.chunk + 1);
    }
    __syncwarp();
  }

  // Drain: every TMA load this warp issued must land before the CTA exits.
  __syncwarp();
  if (lane == 0 && p.use_tma) {
    for (uint32_t s = cm_seq; s < ld_seq; ++s) {
      if (!mbar_wait_bounded(&sm.full[s % STAGES], (s / STAGES) & 1u, p.wait_limit_ns)) {
        record_device_error(MAMBA_ERR_TIMEOUT);
        break;
      }
    }
  }
  __syncwarp();
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
