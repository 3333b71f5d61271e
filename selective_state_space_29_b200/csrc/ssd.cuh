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
// A CTA of four warps owns two heads of one batch row over one super-chunk
// and walks its chunks of 64 tokens in order.  Per chunk and head, all
// products are tcgen05.mma (bf16 operands from shared memory, fp32
// accumulators in tensor memory), issued by one thread:
//   G   = C B^T                     64 x 64, K = N      (same for both heads)
//   Y   = M X + C~ S_in             64 x 64, K = 64 + N  (M = G o e^{a(cum_t - cum_s)} o w_s,
//                                                         masked s > t; C~ = e^{a cum_t} C)
//   dS^T = X^T Bw                   64 x N,  K = 64      (Bw_s = e^{a(cum_end - cum_s)} w_s B_s)
// The M = 64 accumulators of head 0 sit in tensor-memory lanes 0-15 of each
// 32-lane sub-partition and those of head 1 in lanes 16-31, so every thread
// of a warp reads one row of one head: thread i of warp w owns row (or
// channel) 16w + i%16 of head i/16.  The warps turn G into M, form C~ and
// Bw, and run the epilogues: y = Y + D x, and the fp32 state
// S = e^{a cum_end} S + dS, kept in registers (a bf16 copy in shared memory
// is the next chunk's operand).  x, B and C arrive through a ring of
// cp.async copies into the no-swizzle core-matrix layouts the tensor core
// reads (8 rows x 16 bytes per core matrix).
//
// Long sequences with few (batch row, head) pairs are cut into
// super-chunks: an aggregate kernel (the same kernel, state only) runs each
// super-chunk but the last from a zero state and records its end state and
// total decay; the main kernel folds the aggregates of the earlier
// super-chunks into its entering state.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"

namespace mamba {

constexpr int kSsdQ = 64;       // tokens per chunk
constexpr int kSsdP = 64;       // channels per head
constexpr int kSsdWarps = 4;    // one warpgroup per CTA
constexpr int kSsdHeads = 2;    // heads per CTA
constexpr int kSsdTmemCols = 256;  // dS^T in columns [0, 64), Y in [64, 128), G in [128, 192)

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
  int head_pairs;               // ceil(heads / 2)
  int supers;                   // super-chunks per (batch row, head pair)
  int64_t super_len;            // tokens per super-chunk, a multiple of 64
  int euler;                    // input weight dt (exponential Euler) instead of the ZOH weight
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

// 64 consecutive columns (four loads in flight, one wait)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[4][16];
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld16_nowait(taddr + 16 * q, r[q]);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int i = 0; i < 16; ++i) v[16 * q + i] = __uint_as_float(r[q][i]);
}

// N consecutive columns, N a multiple of 16
template <int N>
__device__ __forceinline__ void tmem_ldN(uint32_t taddr, float (&v)[N]) {
  uint32_t r[N / 16][16];
#pragma unroll
  for (int q = 0; q < N / 16; ++q) tmem_ld16_nowait(taddr + 16 * q, r[q]);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < N / 16; ++q)
#pragma unroll
    for (int i = 0; i < 16; ++i) v[16 * q + i] = __uint_as_float(r[q][i]);
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
  static constexpr int kStages = N >= 32 ? 2 : 3;
  static_assert(kStages >= 2, "chunk c+1 must be resident while chunk c is finished");
  static constexpr int kX = kSsdQ * kSsdP * 2;           // one head's x tile (8 KB)
  static constexpr int kBC = kSsdQ * N * 2;              // one B or C tile
  static constexpr int kStage = kSsdHeads * kX + 2 * kBC;  // x of both heads, B, C
  static constexpr int kRing = kStages * kStage;
  static constexpr int kM = kRing;                       // [2 heads] M tiles, 64 x 64
  static constexpr int kCt = kM + kSsdHeads * kSsdQ * kSsdQ * 2;  // [2] C~ tiles, 64 x N
  static constexpr int kBw = kCt + kSsdHeads * kBC;      // [2] Bw tiles, 64 x N
  static constexpr int kS = kBw + kSsdHeads * kBC;       // [2] bf16 state copies, 64 ch x N
  static constexpr int kCum = kS + kSsdHeads * kSsdP * N * 2;  // [2][64] cum (log2), [2][64] w, [2][64] u
  static constexpr int kWsum = kCum + 3 * kSsdHeads * kSsdQ * 4;  // [4 warps][2 heads] partial sums
  static constexpr int kDs = kWsum + kSsdWarps * kSsdHeads * 4;   // [2 heads][64] D
  static constexpr int kBar = kDs + kSsdHeads * kSsdP * 4;        // 2 mbarriers
  static constexpr int kTslot = kBar + 16;
  static constexpr int kBytes = kTslot + 16 + 1024;      // + room to align the base to 1024
  static constexpr int kSboBC = (N / 8) * 128;            // K-major [rows][N]
};

template <int N, bool AGG>
__global__ void __launch_bounds__(kSsdWarps * 32)
ssd_chunk_kernel(const SsdArgs a) {
  using L = SsdSmem<N>;
  static_assert(N % 16 == 0 && N <= 64, "states in steps of 16, at most 64 (tensor-memory columns)");
  extern __shared__ __align__(1024) unsigned char ssd_smem_raw[];
  unsigned char* smem = ssd_smem_raw + ((1024u - (smem_addr(ssd_smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int hd = lane >> 4;                 // head of this thread within the CTA
  const int row = 16 * warp + (lane & 15);  // its row (token) or channel
  const int64_t channels = (int64_t)a.heads * kSsdP;

  // job: (batch row, head pair, super-chunk); the aggregate kernel has one
  // super-chunk fewer per pair
  const int per_seq = AGG ? a.supers - 1 : a.supers;
  const int64_t seq = blockIdx.x / per_seq;  // batch row * head_pairs + pair
  const int j = (int)(blockIdx.x % per_seq);
  const int64_t b = seq / a.head_pairs;
  const int hp = (int)(seq % a.head_pairs);
  const int h = 2 * hp + hd;                // this thread's head
  const bool hok = h < a.heads;
  const bool pair = 2 * hp + 1 < a.heads;   // the CTA's second head exists
  const int64_t t_begin = (int64_t)j * a.super_len;
  const int64_t t_end = t_begin + a.super_len < a.len ? t_begin + a.super_len : a.len;
  const int nchunks = (int)((t_end - t_begin + kSsdQ - 1) / kSsdQ);

  uint64_t* bar_g = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* bar_y = bar_g + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kTslot);
  if (tid == 0) {
    mbar_init(bar_g, 1);
    mbar_init(bar_y, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tslot)),
                 "n"(kSsdTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  griddep_wait();  // inputs (and the aggregates) may come from the previous kernel

  const int hc = hok ? h : 0;               // a valid head for reads
  const float a_h = __ldg(a.A + hc);
  const float a2 = a_h * 1.4426950408889634f;  // a in log2 units
  const __nv_bfloat16* Bg = a.B + (b * a.len) * N;
  const __nv_bfloat16* Cg = a.C + (b * a.len) * N;
  const unsigned short* dtg = reinterpret_cast<const unsigned short*>(a.dt) + (b * a.len) * a.heads + hc;

  // stage one chunk's x (both heads), B (and C) into ring slot `slot`
  auto load_chunk = [&](int c, int slot) {
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    const uint32_t sx = sbase + slot * L::kStage;
#pragma unroll
    for (int i = tid; i < kSsdHeads * kSsdQ * 8; i += kSsdWarps * 32) {
      const int hh = i / (kSsdQ * 8), rem = i % (kSsdQ * 8);
      const int t = rem >> 3, c8 = rem & 7;
      const bool ok = t0 + t < t_end && 2 * hp + hh < a.heads;
      const __nv_bfloat16* src = a.x + (b * a.len + t0 + t) * channels + (int64_t)(2 * hp + hh) * kSsdP + c8 * 8;
      cp_async16(sx + hh * L::kX + (t >> 3) * 1024 + c8 * 128 + (t & 7) * 16, ok ? (const void*)src : (const void*)a.x,
                 ok);
    }
    const uint32_t sb = sx + kSsdHeads * L::kX;
#pragma unroll
    for (int i = tid; i < kSsdQ * (N / 8); i += kSsdWarps * 32) {
      const int t = i / (N / 8), n8 = i % (N / 8);
      const bool ok = t0 + t < t_end;
      const uint32_t off = (t >> 3) * L::kSboBC + n8 * 128 + (t & 7) * 16;
      cp_async16(sb + off, ok ? (const void*)(Bg + (t0 + t) * N + n8 * 8) : (const void*)a.B, ok);
      if (!AGG) cp_async16(sb + L::kBC + off, ok ? (const void*)(Cg + (t0 + t) * N + n8 * 8) : (const void*)a.C, ok);
    }
  };
  auto load_dt = [&](int c) -> float {  // this thread's (token, head) step
    const int64_t t = t_begin + (int64_t)c * kSsdQ + row;
    if (c >= nchunks || t >= t_end) return 0.0f;  // padding tokens: no decay, no input
    return __uint_as_float((uint32_t)__ldg(dtg + t * a.heads) << 16);
  };

  // the state of this thread's (head, channel `row`): N fp32 values
  float S[N];
#pragma unroll
  for (int n = 0; n < N; ++n) S[n] = 0.0f;
  const int64_t sidx = ((b * a.heads + hc) * kSsdP + row) * N;  // (batch, channel, n) offset
  if (!AGG && hok) {
    if (a.h0) {
#pragma unroll
      for (int n = 0; n < N; ++n) S[n] = __ldg(a.h0 + sidx + n);
    }
    // fold in the super-chunks before this one
    const int64_t aseq = b * a.heads + h;
    for (int k = 0; k < j; ++k) {
      const int64_t agg = aseq * (a.supers - 1) + k;
      const float dec = exp2f(__ldg(a.agg_decay + agg));
      const float* as = a.agg_state + (agg * kSsdP + row) * N;
#pragma unroll
      for (int n = 0; n < N; ++n) S[n] = fmaf(dec, S[n], __ldg(as + n));
    }
  }
  // bf16 copy of the state (K-major [channel][n]) for the next chunk's C~ S_in
  auto store_state_copy = [&]() {
    unsigned char* st = smem + L::kS + hd * (kSsdP * N * 2) + (row >> 3) * L::kSboBC + (row & 7) * 16;
#pragma unroll
    for (int n8 = 0; n8 < N / 8; ++n8) {
      uint4 v;
      v.x = pack_bf16(S[8 * n8 + 0], S[8 * n8 + 1]);
      v.y = pack_bf16(S[8 * n8 + 2], S[8 * n8 + 3]);
      v.z = pack_bf16(S[8 * n8 + 4], S[8 * n8 + 5]);
      v.w = pack_bf16(S[8 * n8 + 6], S[8 * n8 + 7]);
      *reinterpret_cast<uint4*>(st + n8 * 128) = v;
    }
  };
  if (!AGG) store_state_copy();

  float* Ds = reinterpret_cast<float*>(smem + L::kDs);  // [2][64] D of both heads (0 without D)
  Ds[hd * kSsdP + row] = (a.D && hok) ? __ldg(a.D + (int64_t)h * kSsdP + row) : 0.0f;
  float* cum_s = reinterpret_cast<float*>(smem + L::kCum);  // [2][64]
  float* w_s = cum_s + kSsdHeads * kSsdQ;                    // [2][64]
  float* u_s = w_s + kSsdHeads * kSsdQ;                      // [2][64] e^{-a cum_s} w_s
  float* wsum = reinterpret_cast<float*>(smem + L::kWsum);   // [4][2]
  float total_log2 = 0.0f;

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t t_lane = tmem + ((uint32_t)(32 * warp) << 16);  // this warp's sub-partition, + lane i = thread
  const uint32_t d_off = (uint32_t)(16 * 1) << 16;                // head 1's accumulators: lanes 16-31

  // Shared-memory descriptors, built once: a K step (or another ring slot /
  // head) only moves the start address, the low 14 bits in 16-byte units
  const uint64_t dBC = umma_desc(sbase, 128, L::kSboBC);      // K-major [rows][N]: C, B, C~, S
  const uint64_t dM = umma_desc(sbase, 128, 1024);            // K-major [64][64]: M
  const uint64_t dX = umma_desc(sbase, 1024, 128);            // MN-major x (B of Y, A of dS^T)
  const uint64_t dBw = umma_desc(sbase, L::kSboBC, 128);      // MN-major Bw (B of dS^T)
  auto at = [](uint64_t d, uint32_t off) { return d + (uint64_t)(off >> 4); };
  constexpr uint32_t kIdG = umma_idesc_bf16(64, 64, 0, 0);
  constexpr uint32_t kIdY = umma_idesc_bf16(64, 64, 0, 1);     // M K-major, x MN-major
  constexpr uint32_t kIdOff = umma_idesc_bf16(64, 64, 0, 0);   // C~ K-major, S K-major
  constexpr uint32_t kIdS = umma_idesc_bf16(64, N, 1, 1);      // x^T MN-major, Bw MN-major
  constexpr uint32_t kColS = 0, kColY = 64, kColG = 128;       // tensor-memory columns
  // G = C B^T of chunk c (slot) into columns [128, 192) of both heads' lanes
  auto issue_g = [&](int slot) {
    const uint32_t ob = slot * L::kStage + kSsdHeads * L::kX;  // B tile, then C tile
#pragma unroll
    for (int hh = 0; hh < kSsdHeads; ++hh) {
      if (hh == 1 && !pair) break;
#pragma unroll
      for (int k = 0; k < N / 16; ++k)
        umma_bf16(tmem + hh * d_off + kColG, at(dBC, ob + L::kBC + k * 256), at(dBC, ob + k * 256), kIdG, k > 0);
    }
    umma_commit(bar_g);
  };

  // prologue: the first kStages chunks, and G of chunk 0
#pragma unroll
  for (int s = 0; s < L::kStages; ++s) {
    if (s < nchunks) load_chunk(s, s);
    cp_async_commit();
  }
  cp_async_wait<L::kStages - 1>();  // chunk 0
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (!AGG && tid == 0 && nchunks > 0) issue_g(0);
  float dt = load_dt(0);
  bool ok_run = true;

  for (int c = 0; c < nchunks && ok_run; ++c) {
    const int slot = c % L::kStages;
    const int64_t t0 = t_begin + (int64_t)c * kSsdQ;
    const float ndt = load_dt(c + 1);
    const uint32_t ox = slot * L::kStage;                 // x tiles of the slot
    const uint32_t ob = ox + kSsdHeads * L::kX;           // B tile
    const uint32_t oc = ob + L::kBC;                      // C tile

    // running log2 decay inside the chunk for this thread's head: an
    // inclusive scan over the 16 lanes of the half-warp, then across warps
    float v = dt * a2;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float nb = __shfl_up_sync(0xffffffffu, v, o, 16);
      if ((lane & 15) >= o) v += nb;
    }
    if ((lane & 15) == 15) wsum[warp * kSsdHeads + hd] = v;
    const float wgt = a.euler ? dt : expm1f(dt * a_h) / a_h;
    __syncthreads();  // the warp sums
    float pre = 0.0f;
    for (int w2 = 0; w2 < warp; ++w2) pre += wsum[w2 * kSsdHeads + hd];
    const float cum = v + pre;
    float cum_end = 0.0f;
    for (int w2 = 0; w2 < kSsdWarps; ++w2) cum_end += wsum[w2 * kSsdHeads + hd];
    total_log2 += cum_end;
    cum_s[hd * kSsdQ + row] = cum;
    w_s[hd * kSsdQ + row] = wgt;
    // the decay from s to t factors as e^{a cum_t} e^{-a cum_s} while the
    // factors stay in range (the chunk decays by less than 2^-100)
    const bool split = cum_end > -100.0f;
    u_s[hd * kSsdQ + row] = split ? ex2_approx(-cum) * wgt : 0.0f;

    // C~ = e^{a cum_t} C_t and Bw = e^{a(cum_end - cum_s)} w_s B_s, row `row` of head hd
    {
      const float fB = ex2_approx(cum_end - cum) * wgt;
      const unsigned char* brow = smem + ob + (row >> 3) * L::kSboBC + (row & 7) * 16;
      // Bw [s][n] as MN-major (N = n, K = s): (s/8) (N/8 128) + (n/8) 128 + (s%8) 16 + (n%8) 2,
      // the same bytes as the K-major [s][n] placement of B
      unsigned char* bwrow = smem + L::kBw + hd * L::kBC + (row >> 3) * L::kSboBC + (row & 7) * 16;
#pragma unroll
      for (int n8 = 0; n8 < N / 8; ++n8) {
        const uint4 bv = *reinterpret_cast<const uint4*>(brow + n8 * 128);
        const uint32_t bw4[4] = {bv.x, bv.y, bv.z, bv.w};
        uint32_t op[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw4[q]));
          op[q] = pack_bf16(f.x * fB, f.y * fB);
        }
        *reinterpret_cast<uint4*>(bwrow + n8 * 128) = make_uint4(op[0], op[1], op[2], op[3]);
      }
      if (!AGG) {
        const float fC = ex2_approx(cum);
        const unsigned char* crow = smem + oc + (row >> 3) * L::kSboBC + (row & 7) * 16;
        unsigned char* ctrow = smem + L::kCt + hd * L::kBC + (row >> 3) * L::kSboBC + (row & 7) * 16;
#pragma unroll
        for (int n8 = 0; n8 < N / 8; ++n8) {
          const uint4 cv = *reinterpret_cast<const uint4*>(crow + n8 * 128);
          const uint32_t cw4[4] = {cv.x, cv.y, cv.z, cv.w};
          uint32_t op[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cw4[q]));
            op[q] = pack_bf16(f.x * fC, f.y * fC);
          }
          *reinterpret_cast<uint4*>(ctrow + n8 * 128) = make_uint4(op[0], op[1], op[2], op[3]);
        }
      }
    }
    __syncthreads();  // cum and w of the chunk are in shared memory

    if (!AGG) {
      // M row `row` of head hd from G: causal mask, decay and input weight
      bool got = mbar_wait_bounded(bar_g, (uint32_t)(c & 1), a.wait_limit_ns);
      got = __all_sync(0xffffffffu, got);  // warp-uniform: the tensor-memory loads are warp-wide
      if (!got) {
        if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
        ok_run = false;
      }
      tc_fence_after();
      const float* cum_h = cum_s + hd * kSsdQ;
      const float* w_h = w_s + hd * kSsdQ;
      const float* u_h = u_s + hd * kSsdQ;
      unsigned char* mrow = smem + L::kM + hd * (kSsdQ * kSsdQ * 2) + (row >> 3) * 1024 + (row & 7) * 16;
      if (ok_run) {
        float g[64];
        tmem_ld64(t_lane + kColG, g);
        if (split) {
          // M[t][s] = G[t][s] e^{a cum_t} (e^{-a cum_s} w_s), s <= t
          const float et = ex2_approx(cum);
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const float4 ua = *reinterpret_cast<const float4*>(u_h + 8 * c8);
            const float4 ub = *reinterpret_cast<const float4*>(u_h + 8 * c8 + 4);
            const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
            uint32_t op[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int s0 = 8 * c8 + 2 * e;
              const float m0 = s0 <= row ? g[s0] * et * uu[2 * e] : 0.0f;
              const float m1 = s0 + 1 <= row ? g[s0 + 1] * et * uu[2 * e + 1] : 0.0f;
              op[e] = pack_bf16(m0, m1);
            }
            *reinterpret_cast<uint4*>(mrow + c8 * 128) = make_uint4(op[0], op[1], op[2], op[3]);
          }
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t op[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int s0 = 8 * c8 + 2 * e;
              const float m0 = s0 <= row ? g[s0] * ex2_approx(cum - cum_h[s0]) * w_h[s0] : 0.0f;
              const float m1 = s0 + 1 <= row ? g[s0 + 1] * ex2_approx(cum - cum_h[s0 + 1]) * w_h[s0 + 1] : 0.0f;
              op[e] = pack_bf16(m0, m1);
            }
            *reinterpret_cast<uint4*>(mrow + c8 * 128) = make_uint4(op[0], op[1], op[2], op[3]);
          }
        }
      }
    }

    // the operands built by the warps, and chunk c+1's copies, are complete:
    // issue Y and dS^T of chunk c, then G of chunk c+1 behind them
    cp_async_wait<L::kStages - 2>();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && ok_run) {
#pragma unroll
      for (int hh = 0; hh < kSsdHeads; ++hh) {
        if (hh == 1 && !pair) break;
        const uint32_t xs = ox + hh * L::kX;
        if (!AGG) {
          const uint32_t dy = tmem + hh * d_off + kColY;
          const uint32_t ms = L::kM + hh * (kSsdQ * kSsdQ * 2);
#pragma unroll
          for (int k = 0; k < kSsdQ / 16; ++k) umma_bf16(dy, at(dM, ms + k * 256), at(dX, xs + k * 2048), kIdY, k > 0);
          const uint32_t cts = L::kCt + hh * L::kBC;
          const uint32_t ss = L::kS + hh * (kSsdP * N * 2);
#pragma unroll
          for (int k = 0; k < N / 16; ++k) umma_bf16(dy, at(dBC, cts + k * 256), at(dBC, ss + k * 256), kIdOff, true);
        }
        const uint32_t bws = L::kBw + hh * L::kBC;
#pragma unroll
        for (int k = 0; k < kSsdQ / 16; ++k)
          umma_bf16(tmem + hh * d_off + kColS, at(dX, xs + k * 2048), at(dBw, bws + k * 2 * L::kSboBC), kIdS, k > 0);
      }
      umma_commit(bar_y);
      if (!AGG && c + 1 < nchunks) issue_g((c + 1) % L::kStages);
    }

    if (ok_run) {
      bool got = mbar_wait_bounded(bar_y, (uint32_t)(c & 1), a.wait_limit_ns);
      got = __all_sync(0xffffffffu, got);
      if (!got) {
        if (lane == 0) record_device_error(MAMBA_ERR_TIMEOUT);
        ok_run = false;
      }
    }
    tc_fence_after();
    if (ok_run) {
      if (!AGG) {
        // y = Y + D x for row `row` of head hd -> bf16 -> 16-byte stores
        const float* Dh = Ds + hd * kSsdP;
        const unsigned char* xrow = smem + ox + hd * L::kX + (row >> 3) * 1024 + (row & 7) * 16;
        const bool store = hok && t0 + row < t_end;
        __nv_bfloat16* yrow = a.y + (b * a.len + t0 + row) * channels + (int64_t)hc * kSsdP;
        float yv[64];
        tmem_ld64(t_lane + kColY, yv);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
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
      // S = e^{a cum_end} S + dS for channel `row` of head hd; its bf16 copy
      // feeds the next chunk's C~ S_in (this chunk's products are done)
      const float dec = ex2_approx(cum_end);
      {
        float ds[N];
        tmem_ldN<N>(t_lane + kColS, ds);
#pragma unroll
        for (int i = 0; i < N; ++i) S[i] = fmaf(dec, S[i], ds[i]);
      }
      if (!AGG) store_state_copy();
    }
    tc_fence_before();
    ok_run = __syncthreads_and(ok_run) != 0;  // slot c is read; every read of Y / dS is done
    // chunk c + kStages into the slot chunk c used
    if (c + L::kStages < nchunks) load_chunk(c + L::kStages, slot);
    cp_async_commit();
    dt = ndt;
  }
  cp_async_wait<0>();

  griddep_launch_dependents();
  if (ok_run && hok) {
    if (AGG) {
      const int64_t agg = (b * a.heads + h) * (a.supers - 1) + j;
      float* as = a.agg_state + (agg * kSsdP + row) * N;
#pragma unroll
      for (int n = 0; n < N; ++n) as[n] = S[n];
      if ((lane & 15) == 0 && warp == 0) a.agg_decay[agg] = total_log2;
    } else if (a.final_state && j == a.supers - 1) {
#pragma unroll
      for (int n = 0; n < N; ++n) a.final_state[sidx + n] = S[n];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kSsdTmemCols) : "memory");
}

}  // namespace mamba
