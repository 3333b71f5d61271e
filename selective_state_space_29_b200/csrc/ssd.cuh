// ssd.cuh -- Mamba-2's restricted scan (one scalar A per head, one step per
// (token, head)) in its chunked matrix form, on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory).
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
// A CTA of four builder warps and one issuing warp owns one head of one
// batch row over one super-chunk and walks its chunks of 64 tokens in order.
// Per chunk, all products are tcgen05.mma (bf16 operands from shared memory,
// fp32 accumulators in tensor memory), issued by one thread of the fifth
// warp while the builders prepare the next chunk:
//   G   = C B^T                     64 x 64, K = N
//   Y   = M X + C~ S_in             64 x 64, K = 64 + N  (M = G o e^{a(cum_t - cum_s)} o w_s,
//                                                         masked s > t; C~ = e^{a cum_t} C)
//   dS^T = X^T Bw                   64 x N,  K = 64      (Bw_s = e^{a(cum_end - cum_s)} w_s B_s)
// With M = 64 an accumulator row m sits in tensor-memory lane 32(m/16) +
// m%16; a second tile can take lanes 32(m/16) + 16 + m%16.  G and Y are each
// issued as two 32-column halves, the first half in the low lanes and the
// second in the high ones, so thread i of warp w owns row 16w + i%16 and
// column half i/16 of both: it reads a half row of G (turned into M) and of
// Y (the y epilogue).  dS^T is issued as two halves of its K (tokens 0-31
// into the low lanes, 32-63 into the high ones); the two threads of a
// channel swap halves of their partial sums (N/2 shuffles) and each keeps
// half of the channel's fp32 state S = e^{a cum_end} S + dS in registers
// (a bf16 copy in shared memory is the next chunk's operand).  The first
// thread of a row forms C~, the second Bw.  x, B and C arrive through a ring
// of cp.async copies into the no-swizzle core-matrix layouts the tensor core
// reads (8 rows x 16 bytes per core matrix).  One head per CTA keeps a CTA
// to 128 tensor-memory columns and about 52 KB of shared memory (N = 16),
// so four CTAs share an SM and their chunk pipelines overlap.
//
// Long sequences with few (batch row, head) pairs are cut into
// super-chunks that run side by side, each from a zero state (the first
// from the initial state); each records its end state H_j and its total
// decay.  A correction kernel then composes the state entering super-chunk
// j, S_in(j) = e^{a sum_{j-1}} S_in(j-1) + H_{j-1} (the scan's monoid with a
// scalar decay), adds its effect e^{a cum_t} C_t . S_in(j) to the outputs
// while that decay is at least 2^-32 (the terms left out are 256 times
// under the fp32 rounding of y), and writes the final state.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"

namespace mamba {

constexpr int kSsdQ = 64;       // tokens per chunk
constexpr int kSsdP = 64;       // channels per head
constexpr int kSsdWarps = 4;    // builder warps (one warpgroup: one per tensor-memory sub-partition)
constexpr int kSsdThreads = (kSsdWarps + 1) * 32;  // + one warp that issues the tensor-core products
constexpr int kSsdTmemCols = 128;  // dS^T in columns [0, 64), Y in [64, 96), G in [96, 128)

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
  float* agg_state;             // (batch*heads, supers, 64, N): super-chunk end state from zero
  float* agg_decay;             // (batch*heads, supers): log2 of its total decay
  int64_t len;
  int heads;
  int supers;                   // super-chunks per (batch row, head)
  int64_t super_len;            // tokens per super-chunk, a multiple of 64
  int euler;                    // input weight dt (exponential Euler) instead of the ZOH weight
  int tma;                      // x, B, C tiles by TMA (5-D core-matrix maps) instead of cp.async
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0: nothing is read, the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// tcgen05 pieces
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, no swizzle: start address, the byte
// distance between core matrices along the leading dimension (LBO) and along
// the stride dimension (SBO), all in 16-byte units; version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3fffu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator,
// M x N, A / B K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int m, int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((int)accumulate)
      : "memory");
}

// the mbarrier completes when every tcgen05.mma this thread issued so far has
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit columns of this thread's tensor-memory lane; the
// registers are valid after tmem_wait_ld (several loads may be in flight)
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// N consecutive columns, N a multiple of 8
template <int N>
__device__ __forceinline__ void tmem_ldN(uint32_t taddr, float (&v)[N]) {
  static_assert(N % 8 == 0, "columns in steps of 8");
  constexpr int Q = N / 16;
  uint32_t r[Q > 0 ? Q : 1][16];
  uint32_t t8[8];
#pragma unroll
  for (int q = 0; q < Q; ++q) tmem_ld16_nowait(taddr + 16 * q, r[q]);
  if constexpr (N % 16 != 0) tmem_ld8_nowait(taddr + 16 * Q, t8);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < Q; ++q)
#pragma unroll
    for (int i = 0; i < 16; ++i) v[16 * q + i] = __uint_as_float(r[q][i]);
  if constexpr (N % 16 != 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[16 * Q + i] = __uint_as_float(t8[i]);
  }
}

// e^z - 1 for z <= 0 without a branch: the Taylor polynomial through z^6
// for |z| <= 1/4 (truncation below 1.2e-8 relative), the hardware exp2
// minus one otherwise (|e^z - 1| > 0.22 there); both are evaluated
__device__ __forceinline__ float ssd_expm1(float z) {
  const float z2 = z * z;
  const float lo = fmaf(z, 1.0f / 6.0f, 0.5f);
  const float hi = fmaf(z2, 1.0f / 720.0f, fmaf(z, 1.0f / 120.0f, 1.0f / 24.0f));
  const float poly = fmaf(z2 * z2, hi, fmaf(z2, lo, z));
  const float viaexp2 = ex2_approx(z * 1.4426950408889634f) - 1.0f;
  return fabsf(z) <= 0.25f ? poly : viaexp2;
}

// named barrier 1 over the four builder warps (the issuer warp is not in it)
__device__ __forceinline__ void builders_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool builders_and(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred ip, op;\n\tsetp.ne.u32 ip, %1, 0;\n\tbar.red.and.pred op, 1, 128, ip;\n\t"
      "selp.u32 %0, 1, 0, op;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// shared-memory layout (bytes), every tile in the no-swizzle core-matrix
// form: a core matrix is 8 rows x 16 bytes, stored contiguously (128 B)
//   K-major [rows][K]:   (r/8) SBO + (k/8) 128 + (r%8) 16 + (k%8) 2,  SBO = K/8 * 128
//   X [tok][ch] as MN-major (N or M = ch, K = tok):
//                        (t/8) 1024 + (c/8) 128 + (t%8) 16 + (c%8) 2
//   Bw [s][n] as MN-major (N = n, K = s):
//                        (s/8) (N/8 * 128) + (n/8) 128 + (s%8) 16 + (n%8) 2
// ---------------------------------------------------------------------------
template <int N>
struct SsdSmem {
  static constexpr int kStages = 3;
  static_assert(kStages >= 2, "chunk c+1 must be resident while chunk c is finished");
  static constexpr int kX = kSsdQ * kSsdP * 2;           // the head's x tile (8 KB)
  static constexpr int kBC = kSsdQ * N * 2;              // one B or C tile
  static constexpr int kStage = kX + 2 * kBC;            // x, B, C
  static constexpr int kRing = kStages * kStage;
  // M, C~ and Bw of two chunks (by chunk parity): the warps build chunk
  // c+1's while the tensor core reads chunk c's
  static constexpr int kMtile = kSsdQ * kSsdQ * 2;
  static constexpr int kM = kRing;                       // [2] M tiles, 64 x 64
  static constexpr int kCt = kM + 2 * kMtile;            // [2] C~ tiles, 64 x N
  static constexpr int kBw = kCt + 2 * kBC;              // [2] Bw tiles, 64 x N
  static constexpr int kS = kBw + 2 * kBC;               // bf16 state copy, 64 ch x N
  static constexpr int kCum = kS + kSsdP * N * 2;        // [64] cum (log2), [64] w, [64] u
  static constexpr int kWsum = kCum + 3 * kSsdQ * 4;     // [4 warps] partial sums
  static constexpr int kDs = kWsum + 16;                 // [64] D
  // mbarriers: G, Y, one per ring slot (TMA), operands ready, drain
  static constexpr int kBar = kDs + kSsdP * 4;
  static constexpr int kTslot = kBar + 8 * (4 + kStages);  // tensor-memory address, then the stop flag
  static constexpr int kBytes = kTslot + 16 + 1024;      // + room to align the base to 1024
  static constexpr int kSboBC = (N / 8) * 128;           // K-major [rows][N]
};

template <int N>
__global__ void __launch_bounds__(kSsdThreads)
ssd_chunk_kernel(const SsdArgs a, const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mb,
                 const __grid_constant__ CUtensorMap mc) {
  using L = SsdSmem<N>;
  static_assert(N % 16 == 0 && N <= 64, "states in steps of 16, at most 64 (tensor-memory columns)");
  constexpr int NH = N / 2;                 // states per thread
  extern __shared__ __align__(1024) unsigned char ssd_smem_raw[];
  unsigned char* smem = ssd_smem_raw + ((1024u - (smem_addr(ssd_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int ch = lane >> 4;                 // column half (and half of the states) of this thread
  const int row = 16 * warp + (lane & 15);  // its row (token) or channel
  const int64_t channels = (int64_t)a.heads * kSsdP;

  // job: (batch row, head, super-chunk)
  const int per_seq = a.supers;
  const int64_t seq = blockIdx.x / per_seq;  // batch row * heads + head
  const int j = (int)(blockIdx.x % per_seq);
  const int64_t b = seq / a.heads;
  const int h = (int)(seq % a.heads);
  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;
  const int nchunks = (int)((t_end - t_begin + kSsdQ - 1) / kSsdQ);

  uint64_t* bar_g = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* bar_y = bar_g + 1;
  uint64_t* bar_full = bar_g + 2;                 // [kStages]: the slot's TMA tiles have landed
  uint64_t* bar_ops = bar_full + L::kStages;      // the builders' operands of a chunk are ready
  uint64_t* bar_drain = bar_ops + 1;              // the issuer's last products have completed
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kTslot);
  volatile int* s_stop = reinterpret_cast<volatile int*>(smem + L::kTslot + 4);  // the builders left early
  const bool builder = warp < kSsdWarps;
  if (tid == 0) {
    mbar_init(bar_g, 1);
    mbar_init(bar_y, 1);
    for (int s2 = 0; s2 < L::kStages; ++s2) mbar_init(bar_full + s2, 1);
    mbar_init(bar_ops, 1);
    mbar_init(bar_drain, 1);
    *s_stop = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tslot)),
                 "n"(kSsdTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  griddep_wait();  // inputs (and the aggregates) may come from the previous kernel

  const float a_h = __ldg(a.A + h);
  const float inv_a = 1.0f / a_h;
  const float a2 = a_h * 1.4426950408889634f;  // a in log2 units
  const __nv_bfloat16* Bg = a.B + (b * a.len) * N;
  const __nv_bfloat16* Cg = a.C + (b * a.len) * N;
  const __nv_bfloat16* xg = a.x + (b * a.len) * channels + (int64_t)h * kSsdP;
  const unsigned short* dtg = reinterpret_cast<const unsigned short*>(a.dt) + (b * a.len) * a.heads + h;

  // Stage one chunk's x, B (and C) into ring slot `slot`.  Piece i of 16
  // bytes: i % 8 is the token within a group of 8, so the 8 lanes of a
  // quarter-warp fill one core matrix (128 contiguous bytes of shared memory,
  // one wavefront), while a warp reads 8 token rows, whole 32-byte sectors.
  auto load_chunk = [&](int c, int slot) {
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    if (a.tma) {  // one thread, three tiles, completion on the slot's barrier
      if (tid == 0) {
        unsigned char* dx = smem + slot * L::kStage;
        mbar_arrive_expect_tx(bar_full + slot, (uint32_t)(L::kX + 2 * L::kBC));
        tma_load_5d(dx, &mx, bar_full + slot, 0, 0, 8 * h, (int)(t0 / 8), (int)b);
        tma_load_5d(dx + L::kX, &mb, bar_full + slot, 0, 0, 0, (int)(t0 / 8), (int)b);
        tma_load_5d(dx + L::kX + L::kBC, &mc, bar_full + slot, 0, 0, 0, (int)(t0 / 8), (int)b);
      }
      return;
    }
    const uint32_t sx = sbase + slot * L::kStage;
#pragma unroll
    for (int i = tid; i < kSsdQ * 8; i += kSsdWarps * 32) {
      const int t = (i & 7) + 8 * (i >> 6), c8 = (i >> 3) & 7;
      const bool ok = t0 + t < t_end;
      const __nv_bfloat16* src = xg + (t0 + t) * channels + c8 * 8;
      cp_async16(sx + (t >> 3) * 1024 + c8 * 128 + (t & 7) * 16, ok ? (const void*)src : (const void*)a.x, ok);
    }
    const uint32_t sb = sx + L::kX;
#pragma unroll
    for (int i = tid; i < kSsdQ * (N / 8); i += kSsdWarps * 32) {
      const int n8 = (i >> 3) % (N / 8), t = (i & 7) + 8 * (i / (8 * (N / 8)));
      const bool ok = t0 + t < t_end;
      const uint32_t off = (t >> 3) * L::kSboBC + n8 * 128 + (t & 7) * 16;
      cp_async16(sb + off, ok ? (const void*)(Bg + (t0 + t) * N + n8 * 8) : (const void*)a.B, ok);
      cp_async16(sb + L::kBC + off, ok ? (const void*)(Cg + (t0 + t) * N + n8 * 8) : (const void*)a.C, ok);
    }
  };
  // this thread's (token, head) step as raw bf16 bits (0 for padding tokens:
  // no decay, no input); widened where it is used, a chunk later, so the
  // load's latency is not waited for when it is issued
  auto load_dt = [&](int c) -> uint32_t {
    const int64_t t = t_begin + (int64_t)c * kSsdQ + row;
    if (c >= nchunks || t >= t_end) return 0u;
    return (uint32_t)__ldg(dtg + t * a.heads);
  };

  // this thread's half of the state of channel `row`: states ch NH ..
  // ch NH + NH - 1, fp32
  float S[NH];
#pragma unroll
  for (int n = 0; n < NH; ++n) S[n] = 0.0f;
  const int64_t sidx = ((b * a.heads + h) * kSsdP + row) * N + ch * NH;  // (batch, channel, n) offset
  if (builder && a.h0 && j == 0) {  // later super-chunks run from zero (the correction kernel adds their carry)
#pragma unroll
    for (int n = 0; n < NH; ++n) S[n] = __ldg(a.h0 + sidx + n);
  }
  // bf16 copy of the state (K-major [channel][n]) for the next chunk's C~ S_in
  auto store_state_copy = [&]() {
    unsigned char* st = smem + L::kS + (row >> 3) * L::kSboBC + (row & 7) * 16;
#pragma unroll
    for (int q = 0; q < NH / 8; ++q) {
      uint4 v;
      v.x = pack_bf16(S[8 * q + 0], S[8 * q + 1]);
      v.y = pack_bf16(S[8 * q + 2], S[8 * q + 3]);
      v.z = pack_bf16(S[8 * q + 4], S[8 * q + 5]);
      v.w = pack_bf16(S[8 * q + 6], S[8 * q + 7]);
      *reinterpret_cast<uint4*>(st + (ch * (NH / 8) + q) * 128) = v;
    }
  };
  if (builder) store_state_copy();

  float* Ds = reinterpret_cast<float*>(smem + L::kDs);  // [64] D of the head (0 without D)
  if (builder && ch == 0) Ds[row] = a.D ? __ldg(a.D + (int64_t)h * kSsdP + row) : 0.0f;
  float* cum_s = reinterpret_cast<float*>(smem + L::kCum);  // [64]
  float* w_s = cum_s + kSsdQ;                                // [64]
  float* u_s = w_s + kSsdQ;                                  // [64] e^{-a cum_s} w_s
  float* wsum = reinterpret_cast<float*>(smem + L::kWsum);   // [4]

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t t_lane = tmem + ((uint32_t)(32 * warp) << 16);  // this warp's sub-partition, + lane i = thread
  const uint32_t d_off = (uint32_t)16 << 16;                     // the second half's tiles: lanes 16-31

  // Shared-memory descriptors, built once: a K step (or another ring slot)
  // only moves the start address, the low 14 bits in 16-byte units
  const uint64_t dBC = umma_desc(sbase, 128, L::kSboBC);      // K-major [rows][N]: C, B, C~, S
  const uint64_t dM = umma_desc(sbase, 128, 1024);            // K-major [64][64]: M
  const uint64_t dX = umma_desc(sbase, 1024, 128);            // MN-major x (B of Y, A of dS^T)
  const uint64_t dBw = umma_desc(sbase, L::kSboBC, 128);      // MN-major Bw (B of dS^T)
  auto at = [](uint64_t d, uint32_t off) { return d + (uint64_t)(off >> 4); };
  constexpr uint32_t kIdG = umma_idesc_bf16(64, 32, 0, 0);     // C K-major, B rows K-major
  constexpr uint32_t kIdY = umma_idesc_bf16(64, 32, 0, 1);     // M K-major, x MN-major
  constexpr uint32_t kIdOff = umma_idesc_bf16(64, 32, 0, 0);   // C~ K-major, S K-major
  constexpr uint32_t kIdS = umma_idesc_bf16(64, N, 1, 1);      // x^T MN-major, Bw MN-major
  constexpr uint32_t kColS = 0, kColY = 64, kColG = 96;        // tensor-memory columns
  // G = C B^T of chunk c (slot): column half hh (s = 32 hh ..) into lanes + 16 hh
  auto issue_g = [&](int slot) {
    const uint32_t ob = slot * L::kStage + L::kX;  // B tile, then C tile
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int k = 0; k < N / 16; ++k)
        umma_bf16(tmem + hh * d_off + kColG, at(dBC, ob + L::kBC + k * 256), at(dBC, ob + 4 * hh * L::kSboBC + k * 256),
                  kIdG, k > 0);
    umma_commit(bar_g);
  };

  // TMA: the tiles of chunk k have landed (bounded wait on the slot's
  // barrier).  Thread 0 counts the chunks it issued and the highest one it
  // saw land, so that it can drain the copies still in flight if the CTA
  // leaves early.
  int n_issued = nchunks < L::kStages ? nchunks : L::kStages, n_landed = 0;
  auto tiles_ready = [&](int k) -> bool {
    if (!a.tma) return true;
    const bool ok = mbar_wait_bounded(bar_full + k % L::kStages, (uint32_t)((k / L::kStages) & 1), a.wait_limit_ns);
    if (ok && k + 1 > n_landed) n_landed = k + 1;
    return ok;
  };
  bool ok_run = true;
  uint32_t dt_raw = load_dt(0);
  float total_log2 = 0.0f;

  // ---- the front of chunk f: Delta scan, C~ and Bw, then M from G (the
  // operands the warps build; buffers f & 1).  Returns the chunk's total
  // log2 decay.
  auto front = [&](int f) -> float {
    const int slot = f % L::kStages;
    const uint32_t ob = slot * L::kStage + L::kX;  // B tile
    const uint32_t oc = ob + L::kBC;               // C tile
    const int pb = f & 1;
    const float dt = __uint_as_float(dt_raw << 16);
    dt_raw = load_dt(f + 1);
    // running log2 decay inside the chunk: an inclusive scan over the 16
    // rows of the half-warp (both halves of a warp hold the same rows), then
    // across warps
    float v = dt * a2;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float nb = __shfl_up_sync(0xffffffffu, v, o, 16);
      if ((lane & 15) >= o) v += nb;
    }
    if (lane == 15) wsum[warp] = v;
    const float wgt = a.euler ? dt : ssd_expm1(dt * a_h) * inv_a;
    // the chunk's tiles are resident: by TMA (the slot's barrier), or by
    // this thread's cp.async groups (the ones of later chunks may still fly;
    // the builders' barrier below makes every thread's copies visible, and
    // the tensor core reads them only after the next fenced bar_ops arrival)
    cp_async_wait<L::kStages - 2>();
    bool landed = tiles_ready(f);
    if (!landed && tid == 0) record_device_error(MAMBA_ERR_TIMEOUT);
    ok_run = builders_and(ok_run && landed);  // the warp sums, the copies, and the vote
    float pre = 0.0f;
    for (int w2 = 0; w2 < warp; ++w2) pre += wsum[w2];
    const float cum = v + pre;
    const float cum_end = (wsum[0] + wsum[1]) + (wsum[2] + wsum[3]);
    // the decay from s to t factors as e^{a cum_t} e^{-a cum_s} while the
    // factors stay in range (the chunk decays by less than 2^-100)
    const bool split = cum_end > -100.0f;
    if (ch == 0) {
      cum_s[row] = cum;
      w_s[row] = wgt;
      u_s[row] = split ? ex2_approx(-cum) * wgt : 0.0f;
    }
    // C~ = e^{a cum_t} C_t and Bw = e^{a(cum_end - cum_s)} w_s B_s for row
    // `row`: each of the row's two threads takes half of the 16-byte pieces
    {
      auto scaled = [&](const unsigned char* src, unsigned char* dst, float fac) {
        const uint4 w = *reinterpret_cast<const uint4*>(src);
        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
        uint32_t op[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[q]));
          op[q] = pack_bf16(x2.x * fac, x2.y * fac);
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(op[0], op[1], op[2], op[3]);
      };
      const uint32_t roff = (row >> 3) * L::kSboBC + (row & 7) * 16;
      // Bw [s][n] as MN-major (N = n, K = s): (s/8) (N/8 128) + (n/8) 128 + (s%8) 16 + (n%8) 2,
      // the same bytes as the K-major [s][n] placement of B
      const float fB = ex2_approx(cum_end - cum) * wgt;
      const float fC = ex2_approx(cum);
#pragma unroll
      for (int q = 0; q < N / 16; ++q) {
        const int n8 = ch * (N / 16) + q;
        scaled(smem + ob + roff + n8 * 128, smem + L::kBw + pb * L::kBC + roff + n8 * 128, fB);
        scaled(smem + oc + roff + n8 * 128, smem + L::kCt + pb * L::kBC + roff + n8 * 128, fC);
      }
    }
    builders_sync();  // cum and w of the chunk are in shared memory
    // M row `row`, columns s = 32 ch .. 32 ch + 31, from G: causal mask,
    // decay and input weight
    bool got = ok_run && mbar_wait_bounded(bar_g, (uint32_t)(f & 1), a.wait_limit_ns);
    got = __all_sync(0xffffffffu, got);  // warp-uniform: the tensor-memory loads are warp-wide
    if (!got && ok_run) {
      if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
      ok_run = false;
    }
    tc_fence_after();
    unsigned char* mrow = smem + L::kM + pb * L::kMtile + (row >> 3) * 1024 + (row & 7) * 16;
    if (ok_run) {
      float g[32];
      tmem_ldN<32>(t_lane + kColG, g);
      const int sb = 32 * ch;
      if (split) {
        // M[t][s] = G[t][s] e^{a cum_t} (e^{-a cum_s} w_s), s <= t
        const float et = ex2_approx(cum);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const float4 ua = *reinterpret_cast<const float4*>(u_s + sb + 8 * c8);
          const float4 ub = *reinterpret_cast<const float4*>(u_s + sb + 8 * c8 + 4);
          const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
          uint32_t op[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int s0 = sb + 8 * c8 + 2 * e, i0 = 8 * c8 + 2 * e;
            const float m0 = s0 <= row ? g[i0] * et * uu[2 * e] : 0.0f;
            const float m1 = s0 + 1 <= row ? g[i0 + 1] * et * uu[2 * e + 1] : 0.0f;
            op[e] = pack_bf16(m0, m1);
          }
          *reinterpret_cast<uint4*>(mrow + (4 * ch + c8) * 128) = make_uint4(op[0], op[1], op[2], op[3]);
        }
      } else {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t op[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int s0 = sb + 8 * c8 + 2 * e, i0 = 8 * c8 + 2 * e;
            const float m0 = s0 <= row ? g[i0] * ex2_approx(cum - cum_s[s0]) * w_s[s0] : 0.0f;
            const float m1 = s0 + 1 <= row ? g[i0 + 1] * ex2_approx(cum - cum_s[s0 + 1]) * w_s[s0 + 1] : 0.0f;
            op[e] = pack_bf16(m0, m1);
          }
          *reinterpret_cast<uint4*>(mrow + (4 * ch + c8) * 128) = make_uint4(op[0], op[1], op[2], op[3]);
        }
      }
    }
    return cum_end;
  };

  // ---- the epilogue of chunk c: y = Y + D x, S = e^{a cum_end} S + dS and its
  // bf16 copy (the next chunk's C~ S_in operand)
  auto epilogue = [&](int c, float cum_end) {
    bool got = ok_run && mbar_wait_bounded(bar_y, (uint32_t)(c & 1), a.wait_limit_ns);
    got = __all_sync(0xffffffffu, got);
    if (!got && ok_run) {
      if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
      ok_run = false;
    }
    tc_fence_after();
    if (!ok_run) return;
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    const uint32_t ox = (c % L::kStages) * L::kStage;
    // this thread's half row of Y and its partial dS^T row: one round
    // trip to tensor memory
    float yv[32], ds[N];
    {
      uint32_t ry[2][16], rs[N / 16][16];
      tmem_ld16_nowait(t_lane + kColY, ry[0]);
      tmem_ld16_nowait(t_lane + kColY + 16, ry[1]);
#pragma unroll
      for (int q = 0; q < N / 16; ++q) tmem_ld16_nowait(t_lane + kColS + 16 * q, rs[q]);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        yv[i] = __uint_as_float(ry[0][i]);
        yv[16 + i] = __uint_as_float(ry[1][i]);
      }
#pragma unroll
      for (int q = 0; q < N / 16; ++q)
#pragma unroll
        for (int i = 0; i < 16; ++i) ds[16 * q + i] = __uint_as_float(rs[q][i]);
    }
    {
      // y = Y + D x for row `row`, channels 32 ch .. 32 ch + 31 -> bf16 ->
      // 16-byte stores
      const float* Dh = Ds + 32 * ch;
      const unsigned char* xrow = smem + ox + (row >> 3) * 1024 + (row & 7) * 16 + 4 * ch * 128;
      const bool store = t0 + row < t_end;
      __nv_bfloat16* yrow = a.y + (b * a.len + t0 + row) * channels + (int64_t)h * kSsdP + 32 * ch;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xrow + c8 * 128);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const float4 da = *reinterpret_cast<const float4*>(Dh + 8 * c8);
        const float4 db = *reinterpret_cast<const float4*>(Dh + 8 * c8 + 4);
        const float dd[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        uint32_t op[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
          const int p = 8 * c8 + 2 * e;
          op[e] = pack_bf16(fmaf(dd[2 * e], xf.x, yv[p]), fmaf(dd[2 * e + 1], xf.y, yv[p + 1]));
        }
        if (store) *reinterpret_cast<uint4*>(yrow + 8 * c8) = make_uint4(op[0], op[1], op[2], op[3]);
      }
    }
    // S = e^{a cum_end} S + dS for channel `row`: this thread holds the
    // partial sum over tokens 32 ch .. of every state; it keeps states
    // ch NH .. and swaps the other half with the row's other thread
    const float dec = ex2_approx(cum_end);
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const float keep = ch ? ds[NH + i] : ds[i];
      const float give = ch ? ds[i] : ds[NH + i];
      S[i] = fmaf(dec, S[i], keep + __shfl_xor_sync(0xffffffffu, give, 16));
    }
    store_state_copy();
  };

  // ---- the pipeline.  The issuer warp (one thread) waits on bar_ops,
  // whose phase 0 means chunk 0's tiles are resident and phase c+1 that the
  // builders have chunk c's operands (M, C~, Bw, the state copy) in shared
  // memory, chunk c+1's tiles resident and chunk c-1's tensor-memory results
  // read; it then issues G(c+1) and chunk c's products.  The builders run,
  // per chunk c, the front of c+1 (while the tensor core works on c), the
  // epilogue of c, a vote, the copies of chunk c + kStages into c's slot
  // and the next bar_ops arrival: they never wait for the issue itself.
  if (!builder) {
    if (lane == 0) {
      bool ok = true;
      auto wait_ops = [&](int phase) -> bool {
        const bool got = mbar_wait_bounded(bar_ops, (uint32_t)(phase & 1), a.wait_limit_ns);
        if (!got) record_device_error(MAMBA_ERR_TIMEOUT);
        tc_fence_after();
        return got && *s_stop == 0;
      };
      if (nchunks > 0 && wait_ops(0)) {
        if (tiles_ready(0)) {
          issue_g(0);
        } else {
          record_device_error(MAMBA_ERR_TIMEOUT);
          ok = false;
        }
        for (int c = 0; c < nchunks && ok; ++c) {
          if (!wait_ops(c + 1)) break;
          if (c + 1 < nchunks) {
            if (tiles_ready(c + 1)) {
              issue_g((c + 1) % L::kStages);
            } else {
              record_device_error(MAMBA_ERR_TIMEOUT);
              ok = false;
            }
          }
          const uint32_t ox = (c % L::kStages) * L::kStage;
          const int pb = c & 1;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            // Y half hh (channels 32 hh ..): M X then + C~ S_in
            const uint32_t dy = tmem + hh * d_off + kColY;
#pragma unroll
            for (int k = 0; k < kSsdQ / 16; ++k)
              umma_bf16(dy, at(dM, L::kM + pb * L::kMtile + k * 256), at(dX, ox + 512 * hh + k * 2048), kIdY, k > 0);
#pragma unroll
            for (int k = 0; k < N / 16; ++k)
              umma_bf16(dy, at(dBC, L::kCt + pb * L::kBC + k * 256), at(dBC, L::kS + 4 * hh * L::kSboBC + k * 256),
                        kIdOff, true);
            // dS^T over tokens 32 hh .. 32 hh + 31
#pragma unroll
            for (int k = 2 * hh; k < 2 * hh + 2; ++k)
              umma_bf16(tmem + hh * d_off + kColS, at(dX, ox + k * 2048),
                        at(dBw, L::kBw + pb * L::kBC + k * 2 * L::kSboBC), kIdS, k > 2 * hh);
          }
          umma_commit(bar_y);
        }
      }
      // every product issued has completed before tensor memory is released
      umma_commit(bar_drain);
      if (!mbar_wait_bounded(bar_drain, 0u, a.wait_limit_ns)) record_device_error(MAMBA_ERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // builders: the first kStages chunks' copies
#pragma unroll
    for (int s2 = 0; s2 < L::kStages; ++s2) {
      if (s2 < nchunks) load_chunk(s2, s2);
      cp_async_commit();
    }
    // one arrival on bar_ops by builder thread 0; a stop flag goes first when
    // the builders are leaving early (the issuer then leaves too)
    auto arrive_ops = [&]() {
      if (tid == 0) {
        if (!ok_run) *s_stop = 1;
        mbar_arrive(bar_ops);
      }
    };
    float cum_end_c = 0.0f;
    if (nchunks > 0) {
      cp_async_wait<L::kStages - 1>();  // chunk 0
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const bool landed = tiles_ready(0);
      if (!landed && tid == 0) record_device_error(MAMBA_ERR_TIMEOUT);
      ok_run = builders_and(ok_run && landed);
      arrive_ops();  // phase 0: G(0) may go
      if (ok_run) {
        cum_end_c = front(0);
        total_log2 += cum_end_c;
        cp_async_wait<0>();  // (chunks 1, 2 for G ahead)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        ok_run = builders_and(ok_run);
        tc_fence_after();
        arrive_ops();  // phase 1: chunk 0's products and G(1) may go
      }
    }
    for (int c = 0; c < nchunks && ok_run; ++c) {
      float cum_end_n = 0.0f;
      if (c + 1 < nchunks) {
        cum_end_n = front(c + 1);
        total_log2 += cum_end_n;
      }
      epilogue(c, cum_end_c);
      // chunk c+2's copies, the operands of c+1 and the state copy are
      // complete; every read of chunk c's slot and of Y / dS is done
      cp_async_wait<0>();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      ok_run = builders_and(ok_run);
      tc_fence_after();
      if (ok_run && c + L::kStages < nchunks) {
        load_chunk(c + L::kStages, c % L::kStages);
        n_issued = c + L::kStages + 1;
      }
      cp_async_commit();
      if (c + 1 < nchunks) arrive_ops();  // phase c+2: chunk c+1's products and G(c+2) may go
      cum_end_c = cum_end_n;
    }
  }
  cp_async_wait<0>();
  if (a.tma && tid == 0)  // (only after a timeout) copies issued but never seen to land
    for (int k = n_landed; k < n_issued; ++k) tiles_ready(k);

  griddep_launch_dependents();
  if (builder && ok_run) {
    if (a.supers > 1) {  // the end state from zero and the total decay, for the correction kernel
      const int64_t agg = (b * a.heads + h) * a.supers + j;
      float* as = a.agg_state + (agg * kSsdP + row) * N + ch * NH;
#pragma unroll
      for (int n = 0; n < NH; ++n) as[n] = S[n];
      if (tid == 0) a.agg_decay[agg] = total_log2;
    } else if (a.final_state) {
#pragma unroll
      for (int n = 0; n < NH; ++n) a.final_state[sidx + n] = S[n];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kSsdTmemCols) : "memory");
}

// ---------------------------------------------------------------------------
// Correction of super-chunks 1..S-1 (one CTA of 128 threads per (batch row,
// head, super-chunk j >= 1)).  Thread (p, half) owns channel p of the head
// and half of each chunk's tokens.  It composes the state entering j from
// the end states and decays the main kernel recorded,
//     S_in = 0;  S_in <- e^{a sum_k} S_in + H_k   for k = 0 .. j-1,
// (H_0 carries the initial state), then walks j's chunks while the carried
// decay e^{a cum} is at least 2^-kSsdFixStopLog2 and adds
//     y_t[p] += e^{a cum_t} sum_n C_t[n] S_in[p][n]
// (cum_t: the sum of dt from the super-chunk's start through t).  The last
// super-chunk's CTA writes the final state e^{a sum_{S-1}} S_in + H_{S-1}.
// The walk stops at 2^-20: y is bf16, so the terms left out are 2^11 times
// under its rounding (the selective scan's bf16 correction stops there too).
// ---------------------------------------------------------------------------
constexpr float kSsdFixStopLog2 = 20.0f;

template <int N>
__global__ void __launch_bounds__(128)
ssd_fix_kernel(const SsdArgs a) {
  __shared__ float s_cum[kSsdQ];      // a cum_t in log2 units
  __shared__ float s_wsum[4];
  __shared__ float s_C[kSsdQ * N];    // the chunk's C rows, fp32
  griddep_wait();  // the main kernel's outputs, end states and decays
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = 32 * (warp & 1) + lane;  // channel of the head (consecutive lanes: consecutive channels)
  const int half = warp >> 1;            // tokens half * 32 .. of a chunk
  const int per = a.supers - 1;
  const int64_t seq = blockIdx.x / per;  // batch row * heads + head
  const int j = 1 + (int)(blockIdx.x % per);
  const int64_t b = seq / a.heads;
  const int h = (int)(seq % a.heads);
  const int64_t channels = (int64_t)a.heads * kSsdP;
  const float a2 = __ldg(a.A + h) * 1.4426950408889634f;

  // the entering state of channel p
  float Sin[N];
#pragma unroll
  for (int n = 0; n < N; ++n) Sin[n] = 0.0f;
  for (int k = 0; k < j; ++k) {
    const int64_t agg = seq * a.supers + k;
    const float dec = exp2f(__ldcg(a.agg_decay + agg));
    const float4* H = reinterpret_cast<const float4*>(a.agg_state + (agg * kSsdP + p) * N);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 v = __ldcg(H + q);
      Sin[4 * q] = fmaf(dec, Sin[4 * q], v.x);
      Sin[4 * q + 1] = fmaf(dec, Sin[4 * q + 1], v.y);
      Sin[4 * q + 2] = fmaf(dec, Sin[4 * q + 2], v.z);
      Sin[4 * q + 3] = fmaf(dec, Sin[4 * q + 3], v.w);
    }
  }
  if (j == a.supers - 1 && a.final_state && half == 0) {
    const int64_t agg = seq * a.supers + j;
    const float dec = exp2f(__ldcg(a.agg_decay + agg));
    const float* H = a.agg_state + (agg * kSsdP + p) * N;
    float* dst = a.final_state + ((b * a.heads + h) * kSsdP + p) * N;
#pragma unroll
    for (int n = 0; n < N; ++n) dst[n] = fmaf(dec, Sin[n], __ldcg(H + n));
  }

  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;
  const unsigned short* dtg = reinterpret_cast<const unsigned short*>(a.dt) + (b * a.len) * a.heads + h;
  const __nv_bfloat16* Cg = a.C + (b * a.len) * N;
  __nv_bfloat16* yg = a.y + (b * a.len) * channels + (int64_t)h * kSsdP + p;
  float carry = 0.0f;  // a cum at the chunk's start, log2 units
  for (int64_t t0 = t_begin; t0 < t_end && carry >= -kSsdFixStopLog2; t0 += kSsdQ) {
    const int nt = t_end - t0 < kSsdQ ? (int)(t_end - t0) : kSsdQ;
    __syncthreads();  // the previous chunk's rows are no longer read
    // the chunk's running decay (threads 0..63, one token each) and C rows
    if (tid < kSsdQ) {
      float v = tid < nt ? __uint_as_float((uint32_t)__ldg(dtg + (t0 + tid) * a.heads) << 16) * a2 : 0.0f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float nb = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += nb;
      }
      if (lane == 31) s_wsum[warp] = v;
      s_cum[tid] = v;
    }
    for (int i = tid; i < kSsdQ * N; i += 128) {
      const int t = i / N;
      s_C[i] = t < nt ? __bfloat162float(Cg[(t0 + t) * N + (i - t * N)]) : 0.0f;
    }
    __syncthreads();
    const float w0 = s_wsum[0];
    // the 32 outputs of this thread's half of the chunk: loads all issued
    // first, then the arithmetic, then the stores
    float yv[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int t = 32 * half + r;
      yv[r] = t < nt ? __bfloat162float(yg[(t0 + t) * channels]) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int t = 32 * half + r;
      const float cum = carry + s_cum[t] + (half ? w0 : 0.0f);
      float acc = 0.0f;
#pragma unroll
      for (int n = 0; n < N; ++n) acc = fmaf(s_C[t * N + n], Sin[n], acc);
      if (t < nt) yg[(t0 + t) * channels] = __float2bfloat16_rn(yv[r] + ex2_approx(cum) * acc);
    }
    carry += w0 + (nt > 32 ? s_wsum[1] : 0.0f);
  }
}

}  // namespace mamba
