// mamba_ssm.cu -- C ABI entry points: argument checks, planning of the
// chunked scan, tensor-map set-up, stream-ordered scratch and launches.
// Every arithmetic step of the path runs in the kernels of scan.cuh and
// decode.cuh; nothing here touches tensor data on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "mamba_ssm.h"
#include "common.cuh"
#include "backward.cuh"
#include "decode.cuh"
#include "scan.cuh"
#include "ssd.cuh"
#include "complex_scan.cuh"

namespace mamba {

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait

int elem_size(int dtype) { return dtype == MAMBA_BF16 ? 2 : 4; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// --- device properties, cached per device ---------------------------------
struct DeviceInfo {
  int sms = 0;
  bool ok = false;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

int current_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAMBA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev[dev].ok) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MAMBA_ERR_CUDA;
    g_dev[dev].sms = v;
    g_dev[dev].ok = true;
  }
  *sms = g_dev[dev].sms;
  return MAMBA_OK;
}

// --- stream-ordered scratch -------------------------------------------------
// Scratch comes from a memory pool the library owns on each device, which
// keeps up to kPoolKeepBytes of freed memory across synchronisations: the
// device's default pool returns freed memory to the system at every
// synchronisation, and mapping it again on the next call costs host time
// during which the GPU waits.  Inside a stream capture the allocation is a
// plain cudaMallocAsync (a graph memory node).
constexpr uint64_t kPoolKeepBytes = uint64_t(1) << 30;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[64] = {};

std::atomic<int64_t> g_scratch_allocs{0};  // scratch allocations made by this process

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t stream) {
  g_scratch_allocs.fetch_add(1);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return cudaErrorUnknown;
  int dev = 0;
  if (cs != cudaStreamCaptureStatusNone || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return cudaMallocAsync(p, bytes, stream);
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (!g_pool[dev]) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaMemPool_t np = nullptr;
      if (cudaMemPoolCreate(&np, &props) != cudaSuccess) return cudaMallocAsync(p, bytes, stream);
      uint64_t keep = kPoolKeepBytes;
      cudaMemPoolSetAttribute(np, cudaMemPoolAttrReleaseThreshold, &keep);
      g_pool[dev] = np;
    }
    pool = g_pool[dev];
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, stream);
}

// --- tensor maps through the driver entry point (no link to libcuda) -------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows][cols] array, box [box_rows][box_cols].
bool make_map_2d(CUtensorMap* m, const void* base, int dtype, uint64_t cols, uint64_t rows, uint32_t box_cols,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)elem_size(dtype)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      dtype == MAMBA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D map that lands a [64 tokens][8 g] tile of a bf16 [batch][len][row]
// array in the tensor core's no-swizzle core-matrix layout: dimensions
// (8 elements, token % 8, row / 8, token / 8, batch row), box (8, 8, g, 8, 1)
// walked innermost first, so the tile's byte offset of (token t, element e)
// is (t/8) (128 g) + (e/8) 128 + (t%8) 16 + (e%8) 2.  Needs len % 8 == 0 (the
// token split stays inside a batch row) and row % 8 == 0.
bool make_map_core_tiles(CUtensorMap* m, const void* base, uint64_t row, uint64_t len, uint64_t batch, uint32_t g) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || row % 8 != 0 || len % 8 != 0 || len < 64) return false;
  const cuuint64_t dims[5] = {8, 8, row / 8, len / 8, batch};
  const cuuint64_t strides[4] = {row * 2, 16, 8 * row * 2, len * row * 2};
  const cuuint32_t box[5] = {8, 8, g, 8, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --- scan configuration per element type and state count -------------------
// A CTA is CW consumer warps (4: one per SM sub-partition; 8: two) and one
// producer warp; a consumer's ring holds kStages tiles of kTile tokens (the
// ring of four consumers fits the 227 KB of shared memory of a CTA).
// With R inputs per token (multi-input multi-output) a tile holds 1/R as
// many tokens, so that its u, B and C' rows stay the same size.  With eight
// consumer warps tiles are half as long and the ring two deep, so that
// eight rings fit the shared memory of a CTA.
template <typename TIO, int NS, int R = 1, int CW = 4>
struct ScanCfg {
  static_assert(CW == 4 || CW == 8, "one or two consumer warps per sub-partition");
  static constexpr bool kBf16 = sizeof(TIO) == 2;
  static constexpr int kTile = (kBf16 ? 64 : 32) / R / (CW / 4);
  static constexpr int kStages = (CW == 8 || (kBf16 && NS >= 32)) ? 2 : 3;
};
#ifndef MAMBA_SCAN_JOBS_PER_WARP
#define MAMBA_SCAN_JOBS_PER_WARP 8
#endif
constexpr int kJobsPerWarp = MAMBA_SCAN_JOBS_PER_WARP;  // chunks per consumer warp, for dynamic balance
// With eight consumers (very long super-chunks) the jobs are twice as many
// and as short (measured at 2^20 tokens x 2048 channels: 8.47 ms with 8 jobs
// per warp, 8.19 with 16, 8.23 with 32); with four consumers more jobs cost
// more hand-offs than they gain in balance.
#ifndef MAMBA_SCAN_JOBS_PER_WARP_CW8
#define MAMBA_SCAN_JOBS_PER_WARP_CW8 (2 * MAMBA_SCAN_JOBS_PER_WARP)
#endif
constexpr int kJobsPerWarpCw8 = MAMBA_SCAN_JOBS_PER_WARP_CW8;
// Super-chunks of at most 2,048 tokens are cut into half as many jobs: their
// chunks are short already (measured on 2048 channels: 2^14 tokens, 1,664-
// token super-chunks, 0.262 -> 0.254 ms; 2^15 unchanged; 2^16 slower).
constexpr int64_t kShortSuperChunk = 2048;
// streams (channel group x super-chunk) per resident consumer warp, in percent,
// below which sequences are cut into super-chunks
#ifndef MAMBA_SCAN_STREAMS_PCT
#define MAMBA_SCAN_STREAMS_PCT 100
#endif
constexpr int64_t kStreamsPerWarpPct = MAMBA_SCAN_STREAMS_PCT;

struct Plan {
  int groups_d = 0;         // ceil(channels / 32)
  int64_t groups = 0;       // batch * groups_d
  int cw = 4;               // consumer warps per CTA
  int warps_total = 0;      // resident consumer warps: SMs * cw
  int supers = 1;
  int64_t super_len = 0;
  int64_t chunk_len = 0;
  int chunks_full = 1, chunks_last = 1;
};

// How a scan is laid out and split.  Every consumer warp needs a stream of
// its own (a 32-channel group over a stretch of time); when the groups are
// fewer than the resident consumer warps, sequences are cut into
// super-chunks that run from zero side by side and are joined afterwards by
// the correction kernel (about as many streams as warps: each extra
// super-chunk adds a correction walk, which ends once the carried decay is
// below 2^-32).  Within a stream the sequence is cut into chunks so that
// there are about kJobsPerWarp jobs per warp for dynamic balance, each at
// least two tiles long.  A positive `user_chunk` forces super-chunks of that
// length.
Plan plan_scan(int64_t batch, int64_t len, int64_t channels, int sms, int tile, int64_t user_chunk, int cw = 4) {
  Plan pl;
  pl.cw = cw;
  pl.warps_total = sms * cw;
  pl.groups_d = (int)((channels + kCPW - 1) / kCPW);
  pl.groups = batch * pl.groups_d;
  const int64_t groups = std::max<int64_t>(1, pl.groups);
  if (user_chunk > 0) {
    pl.super_len = std::min<int64_t>(user_chunk, len);
  } else {
    int64_t s = 1;
    const int64_t want = (int64_t)pl.warps_total * kStreamsPerWarpPct / 100;  // streams wanted
    if (groups < want) s = (want + groups - 1) / groups;
    s = std::min<int64_t>(s, std::max<int64_t>(1, len / (4 * tile)));
    pl.super_len = (len + s - 1) / s;
    pl.super_len = ((pl.super_len + tile - 1) / tile) * tile;
  }
  pl.super_len = std::max<int64_t>(1, pl.super_len);
  pl.supers = (int)((len + pl.super_len - 1) / pl.super_len);
  const int64_t streams = (int64_t)pl.supers * groups;
  const int64_t jobs_per_warp = cw == 8 ? kJobsPerWarpCw8
                                        : (pl.supers > 1 && pl.super_len <= kShortSuperChunk ? kJobsPerWarp / 2
                                                                                              : kJobsPerWarp);
  int64_t k = (jobs_per_warp * pl.warps_total + streams - 1) / streams;
  k = std::max<int64_t>(1, std::min<int64_t>(k, pl.super_len / (2 * tile)));
  int64_t cl = (pl.super_len + k - 1) / k;
  cl = ((cl + tile - 1) / tile) * tile;
  pl.chunk_len = std::max<int64_t>(1, std::min<int64_t>(cl, pl.super_len));
  pl.chunks_full = (int)((pl.super_len + pl.chunk_len - 1) / pl.chunk_len);
  const int64_t last_len = len - (int64_t)(pl.supers - 1) * pl.super_len;
  pl.chunks_last = (int)((last_len + pl.chunk_len - 1) / pl.chunk_len);
  return pl;
}

struct ScratchLayout {
  size_t ctr, done, fix_segs, ring, ring_sd, agg_h, agg_sd, cum, cs, bs, chan, total;
  int64_t segs_max;  // correction segments of a full super-chunk
};

// widen_b: bf16 data, whose B rows the pre-pass widens to fp32 in scratch
ScratchLayout scratch_layout(const Plan& pl, int ns, int64_t batch, int64_t len, int tile, bool widen_b,
                             int ranks = 1) {
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  const int64_t S = pl.supers;
  const int64_t streams = S * pl.groups;
  const int64_t aggs = S > 1 ? streams : 0;  // aggregates, segment sums: only with super-chunks
  ScratchLayout s;
  const int64_t seg = (int64_t)kFixSegTiles * tile;
  s.segs_max = (pl.super_len + seg - 1) / seg;
  s.ctr = al(4 * sizeof(int));
  s.done = al(sizeof(int) * (size_t)streams);
  s.fix_segs = al(sizeof(int) * (size_t)aggs);
  s.ring = al(sizeof(float) * (size_t)streams * 2 * kCPW * ns);
  s.ring_sd = al(sizeof(float) * (size_t)streams * 2 * kCPW);
  s.agg_h = al(sizeof(float) * (size_t)aggs * kCPW * ns);
  s.agg_sd = al(sizeof(float) * (size_t)aggs * kCPW);
  s.cum = al(sizeof(float) * (size_t)aggs * (size_t)s.segs_max * kCPW);
  s.cs = al(sizeof(float) * (size_t)batch * (size_t)len * (size_t)ranks * (size_t)ns);
  s.bs = widen_b ? s.cs : 0;
  s.chan = al(sizeof(float) * 4 * (size_t)pl.groups_d * (size_t)kCPW);
  s.total = s.ctr + s.done + s.fix_segs + s.ring + s.ring_sd + s.agg_h + s.agg_sd + s.cum + s.cs + s.bs + s.chan;
  return s;
}

int64_t full_jobs(const Plan& pl) {
  const int64_t streams = (int64_t)pl.supers * pl.groups;
  const int64_t streams_early = (int64_t)(pl.supers - 1) * pl.groups;  // super-chunks 0..S-2
  return (int64_t)pl.chunks_last * streams + (int64_t)(pl.chunks_full - pl.chunks_last) * streams_early;
}

int tile_for(int dtype, int cw = 4) {
  if (cw == 8) return dtype == MAMBA_BF16 ? ScanCfg<__nv_bfloat16, 16, 1, 8>::kTile : ScanCfg<float, 16, 1, 8>::kTile;
  return dtype == MAMBA_BF16 ? ScanCfg<__nv_bfloat16, 16>::kTile : ScanCfg<float, 16>::kTile;
}

// Consumer warps for a scan.  Two per sub-partition hide more of a token's
// latency but need twice the streams, i.e. twice the super-chunks, each of
// which adds a correction walk of ~1,500 tokens, and halve the tile, i.e.
// double the barrier traffic per token; that pays off only for bf16 data
// in very long super-chunks (measured on 2048 channels: 2-4% faster at 2^20
// tokens, even at 2^19, slower at 2^18 and below, and 50% slower for fp32
// data, whose 16-token tiles hide too little of the load latency).  Built
// for the zero-order-hold scan with one input and 16 states (`eligible`);
// a forced chunk length keeps four.
#ifndef MAMBA_LONG_SUPER_CHUNK
#define MAMBA_LONG_SUPER_CHUNK 65536
#endif
constexpr int64_t kLongSuperChunk = MAMBA_LONG_SUPER_CHUNK;
Plan choose_plan(int64_t batch, int64_t len, int64_t channels, int64_t nstate, int sms, int dtype,
                 int64_t user_chunk, bool eligible) {
  Plan pl = plan_scan(batch, len, channels, sms, tile_for(dtype), user_chunk);
  if (eligible && dtype == MAMBA_BF16 && nstate == 16 && user_chunk == 0 && pl.supers > 1 &&
      pl.super_len >= kLongSuperChunk)
    pl = plan_scan(batch, len, channels, sms, tile_for(dtype, 8), 0, 8);
  return pl;
}

// state counts the kernels are built for
template <typename F>
int dispatch_nstate(int64_t nstate, F&& f) {
  switch (nstate) {
    case 4: return f(std::integral_constant<int, 4>{});
    case 8: return f(std::integral_constant<int, 8>{});
    case 16: return f(std::integral_constant<int, 16>{});
    case 32: return f(std::integral_constant<int, 32>{});
    default: return MAMBA_ERR_UNSUPPORTED;
  }
}

// pre-pass, chunked scan, and the correction kernel when there are super-chunks
int64_t kernels_per_call(const Plan& pl) { return pl.supers > 1 ? 3 : 2; }

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes; it waits for that kernel's
// writes (griddepcontrol.wait) before it reads or writes global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Scratch for mamba_selective_scan_noalloc.
//
// Some callers may not allocate device memory inside an operation: inference
// runtimes and plugin hosts that plan every byte of device memory ahead of
// time and hand operations only their inputs and outputs, deployments with a
// fixed, audited memory budget, and processes whose device memory is held by
// another allocator (a framework's caching pool), where a driver allocation
// can fail at an arbitrary point.  For them the scan's scratch (job counters,
// the chunk-to-chunk state hand-off, super-chunk aggregates and C/(n+1))
// lives in one file-scope device array of fixed size, reserved on every GPU
// that loads the library for as long as the process lives.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol, so the address is looked
// up once per device (with that device current) and cached.
int noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAMBA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return MAMBA_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return MAMBA_OK;
}

// Enqueue one scan with the given plan on caller-provided scratch (laid out
// by scratch_layout): pre-pass, chunked pass, [correction].  R > 1: the
// multi-input multi-output scan (u, y [batch][len][R][channels], B, C
// [batch][len][R][nstate]).
template <typename TIO, int NS, int METHOD, bool CKPT = false, int R = 1, int CW = 4>
int launch_scan_on(const void* u, const void* delta, const float* A, const void* B, const void* C, const float* D,
                   const float* h0, void* y, float* final_state, int64_t batch, int64_t len, int64_t channels,
                   unsigned flags, int dtype, cudaStream_t stream, const Plan& pl, int sms,
                   unsigned char* scratch, float* ckpt = nullptr) {
  constexpr int TILE = ScanCfg<TIO, NS, R, CW>::kTile;
  constexpr int STAGES = ScanCfg<TIO, NS, R, CW>::kStages;
  constexpr bool kWidenB = sizeof(TIO) == 2;
  const ScratchLayout sl = scratch_layout(pl, NS, batch, len, TILE, kWidenB, R);
  unsigned char* cur = scratch;
  int* counters = reinterpret_cast<int*>(cur); cur += sl.ctr;
  int* done = reinterpret_cast<int*>(cur); cur += sl.done;
  int* fix_segs = reinterpret_cast<int*>(cur); cur += sl.fix_segs;
  float* ring = reinterpret_cast<float*>(cur); cur += sl.ring;
  float* ring_sd = reinterpret_cast<float*>(cur); cur += sl.ring_sd;
  float* agg_h = reinterpret_cast<float*>(cur); cur += sl.agg_h;
  float* agg_sd = reinterpret_cast<float*>(cur); cur += sl.agg_sd;
  float* cum = reinterpret_cast<float*>(cur); cur += sl.cum;
  float* cs = reinterpret_cast<float*>(cur); cur += sl.cs;
  float* bs = kWidenB ? reinterpret_cast<float*>(cur) : nullptr; cur += sl.bs;
  float4* chan = reinterpret_cast<float4*>(cur);

  // tile loads through TMA when every operand can be described by a tensor map
  const size_t es = sizeof(TIO);
  // (B rows are read as fp32: the input itself, or its widened copy)
  const void* b32 = kWidenB ? static_cast<const void*>(bs) : B;
  bool tma = aligned(u, 16) && aligned(delta, 16) && aligned(b32, 16) && (channels * (int64_t)es) % 16 == 0 &&
             (NS * sizeof(float)) % 16 == 0 && encode_fn() != nullptr;
  CUtensorMap mu, mdl, mb, mc;
  std::memset(&mu, 0, sizeof(mu));
  std::memset(&mdl, 0, sizeof(mdl));
  std::memset(&mb, 0, sizeof(mb));
  std::memset(&mc, 0, sizeof(mc));
  if (tma) {
    const uint64_t rows = (uint64_t)batch * (uint64_t)len;
    tma = make_map_2d(&mu, u, dtype, (uint64_t)channels, rows * R, kCPW, TILE * R) &&
          make_map_2d(&mdl, delta, dtype, (uint64_t)channels, rows, kCPW, TILE) &&
          make_map_2d(&mb, b32, MAMBA_F32, NS, rows * R, NS, TILE * R) &&
          make_map_2d(&mc, cs, MAMBA_F32, NS, rows * R, NS, TILE * R);
  }

  ScanParams p;
  std::memset(&p, 0, sizeof(p));
  p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.cs = cs; p.chan = chan; p.h0 = h0; p.y = y;
  p.final_state = final_state;
  p.ckpt = ckpt;
  p.ring = ring; p.ring_sd = ring_sd; p.agg_h = agg_h; p.agg_sd = agg_sd; p.cum = cum; p.fix_segs = fix_segs;
  p.segs_max = (int)sl.segs_max;
  p.fix_vec = (aligned(delta, 16) && aligned(y, 16) && aligned(C, 16) && (channels * (int64_t)es) % 16 == 0 &&
               (NS * es) % 16 == 0)
                  ? 1
                  : 0;
  p.batch = batch; p.len = len; p.channels = channels;
  p.groups_d = pl.groups_d; p.groups = (int)pl.groups;
  p.supers = pl.supers; p.super_len = pl.super_len; p.chunk_len = pl.chunk_len;
  p.chunks_full = pl.chunks_full; p.chunks_last = pl.chunks_last;
  p.use_tma = tma ? 1 : 0;
  p.wait_limit_ns = kWaitLimitNs;

  constexpr size_t smem = scan_smem_bytes<TIO, NS, TILE, STAGES, CW, R>();
  static_assert(smem <= 232448, "scan CTA exceeds the shared memory of an SM");
  auto kern = scan_chunks_kernel<TIO, NS, CW, TILE, STAGES, METHOD, CKPT, R>;
  {
    // the dynamic shared-memory limit is a per-device attribute of the kernel
    static std::mutex mu_attr;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAMBA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu_attr);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MAMBA_ERR_CUDA;
      attr_set[dev] = true;
    }
  }

  const int64_t S = pl.supers;
  const int64_t streams = S * pl.groups;
  const int64_t jobs = full_jobs(pl);
  const int64_t fix_phases = std::min<int64_t>(sl.segs_max, kFixPhases);
  const int64_t fix_warps = (S - 1) * pl.groups * fix_phases;
  if (jobs > 0x7fffffff || streams > 0x7fffffff || fix_warps > 0x7fffffffLL || sl.segs_max > 0x7fffffff)
    return MAMBA_ERR_UNSUPPORTED;
  p.streams = (int)streams;
  p.jobs = (int)jobs;
  p.counters = counters;
  p.done = done;

  // pre-pass: zero the counters and progress flags, C' = C / (n+1) in fp32,
  // B in fp32 (bf16 data), and the per-channel constants
  {
    const int64_t zero_words = (int64_t)((sl.ctr + sl.done + sl.fix_segs) / sizeof(int));
    const int64_t total_c = batch * len * R * NS;
    const int64_t chan_padded = (int64_t)pl.groups_d * kCPW;
    const int64_t total = zero_words + total_c / 4 + chan_padded;  // (four C and B elements per thread)
    if ((total + 255) / 256 > 0x7fffffff) return MAMBA_ERR_UNSUPPORTED;
    scan_prep_kernel<TIO, NS><<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(
        counters, zero_words, static_cast<const TIO*>(C), cs, static_cast<const TIO*>(B), bs, total_c, A, D, chan,
        channels, chan_padded,
        (flags & MAMBA_SCAN_GENERAL_A) ? 1 : 0);
    if (cudaGetLastError() != cudaSuccess) return MAMBA_ERR_CUDA;
  }
  // one persistent pass over every super-chunk from zero (super-chunk 0
  // from the initial state) ...
  const int64_t ctas = std::min<int64_t>(sms, (jobs + CW - 1) / CW);
  if (launch_pdl(kern, dim3((unsigned)ctas), dim3((CW + 1) * 32), smem, stream, p, mu, mdl, mb, mc) !=
      cudaSuccess)
    return MAMBA_ERR_CUDA;
  // ... then the states entering super-chunks 1..S-1 and their effect on y
  // (and on the checkpoints), and the final state
  if (S > 1) {
    const int phases = (int)fix_phases;
    const int64_t blocks = (fix_warps + kFixWarps - 1) / kFixWarps;
    constexpr int fix_smem = kFixWarps * fix_stage_bytes<TIO, NS, TILE, R>();
    if constexpr (fix_smem > 48 * 1024) {
      if (cudaFuncSetAttribute(scan_fix_kernel<TIO, NS, TILE, CKPT, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fix_smem) != cudaSuccess)
        return MAMBA_ERR_CUDA;
    }
    if (launch_pdl(scan_fix_kernel<TIO, NS, TILE, CKPT, R>, dim3((unsigned)blocks), dim3(kFixWarps * 32), fix_smem,
                   stream, p, phases) != cudaSuccess)
      return MAMBA_ERR_CUDA;
  }
  return MAMBA_OK;
}

// The eight-consumer scan exists for 16 states only (choose_plan)
template <typename TIO, int NS>
int launch_cw8(const void* u, const void* delta, const float* A, const void* B, const void* C, const float* D,
               const float* h0, void* y, float* final_state, int64_t batch, int64_t len, int64_t channels,
               unsigned flags, int dtype, cudaStream_t stream, const Plan& pl, int sms, unsigned char* scratch) {
  if constexpr (NS == 16)
    return launch_scan_on<TIO, NS, kZOH, false, 1, 8>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels,
                                                      flags, dtype, stream, pl, sms, scratch);
  else
    return MAMBA_ERR_UNSUPPORTED;
}

// Plan, get scratch (stream-ordered allocation, or the fixed array when
// `noalloc`), enqueue, release the allocation.
template <typename TIO, int NS>
int launch_scan(const void* u, const void* delta, const float* A, const void* B, const void* C, const float* D,
                const float* h0, void* y, float* final_state, int64_t batch, int64_t len, int64_t channels,
                int64_t user_chunk, unsigned flags, int dtype, cudaStream_t stream, bool noalloc,
                float* ckpt = nullptr) {
  int sms = 0;
  if (int st = current_sms(&sms)) return st;
  const bool zoh = !(flags & (MAMBA_SCAN_EULER | MAMBA_SCAN_TRAPEZOID));
  const Plan pl = choose_plan(batch, len, channels, NS, sms, dtype, user_chunk, zoh && !ckpt);
  if (pl.groups > (1 << 30)) return MAMBA_ERR_UNSUPPORTED;
  const ScratchLayout sl = scratch_layout(pl, NS, batch, len, tile_for(dtype, pl.cw), sizeof(TIO) == 2);
  unsigned char* scratch = nullptr;
  if (noalloc) {
    if (sl.total > kNoAllocScratchBytes) return MAMBA_ERR_UNSUPPORTED;  // needs more than the fixed array
    void* base = nullptr;
    if (int st = noalloc_scratch_address(&base)) return st;
    scratch = static_cast<unsigned char*>(base);
  } else {
    if (scratch_alloc(reinterpret_cast<void**>(&scratch), sl.total, stream) != cudaSuccess) return MAMBA_ERR_CUDA;
  }
  int status;
  if (flags & MAMBA_SCAN_EULER)
    status = launch_scan_on<TIO, NS, kEuler>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels, flags,
                                             dtype, stream, pl, sms, scratch);
  else if (flags & MAMBA_SCAN_TRAPEZOID)
    status = launch_scan_on<TIO, NS, kTrapezoid>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels,
                                                 flags, dtype, stream, pl, sms, scratch);
  else if (ckpt)
    status = launch_scan_on<TIO, NS, kZOH, true>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels,
                                                 flags, dtype, stream, pl, sms, scratch, ckpt);
  else if (pl.cw == 8)
    status = launch_cw8<TIO, NS>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels, flags, dtype, stream,
                                 pl, sms, scratch);
  else
    status = launch_scan_on<TIO, NS, kZOH>(u, delta, A, B, C, D, h0, y, final_state, batch, len, channels, flags,
                                           dtype, stream, pl, sms, scratch);
  if (!noalloc && cudaFreeAsync(scratch, stream) != cudaSuccess && status == MAMBA_OK) return MAMBA_ERR_CUDA;
  return status;
}

// The multi-input multi-output scan: plan, stream-ordered scratch, enqueue.
template <typename TIO, int NS, int R>
int launch_scan_mimo(const void* u, const void* delta, const float* A, const void* B, const void* C,
                     const float* D, const float* h0, void* y, float* final_state, int64_t batch, int64_t len,
                     int64_t channels, unsigned flags, int dtype, cudaStream_t stream) {
  int sms = 0;
  if (int st = current_sms(&sms)) return st;
  const Plan pl = plan_scan(batch, len, channels, sms, ScanCfg<TIO, NS, R>::kTile, 0);
  if (pl.groups > (1 << 30)) return MAMBA_ERR_UNSUPPORTED;
  const ScratchLayout sl = scratch_layout(pl, NS, batch, len, ScanCfg<TIO, NS, R>::kTile, sizeof(TIO) == 2, R);
  unsigned char* scratch = nullptr;
  if (scratch_alloc(reinterpret_cast<void**>(&scratch), sl.total, stream) != cudaSuccess) return MAMBA_ERR_CUDA;
  const int status = launch_scan_on<TIO, NS, kZOH, false, R>(u, delta, A, B, C, D, h0, y, final_state, batch, len,
                                                             channels, flags, dtype, stream, pl, sms, scratch);
  if (cudaFreeAsync(scratch, stream) != cudaSuccess && status == MAMBA_OK) return MAMBA_ERR_CUDA;
  return status;
}

// ---------------------------------------------------------------------------
// Host-resident data: the sequence is cut into time pieces; piece k's
// host->device copies, scan and device->host copy of y run on stream k % 2,
// so one piece's copies overlap the neighbouring pieces' scans (the two copy
// directions use separate copy engines).  Piece k resumes from piece k-1's
// final state (an event orders the two streams), which is the same
// recurrence as one scan over the whole sequence.
// ---------------------------------------------------------------------------
std::mutex g_aux_mu;
cudaStream_t g_aux_stream[64] = {};

int aux_stream(cudaStream_t* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAMBA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_aux_mu);
  if (!g_aux_stream[dev] && cudaStreamCreateWithFlags(&g_aux_stream[dev], cudaStreamNonBlocking) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  *out = g_aux_stream[dev];
  return MAMBA_OK;
}

// Rows [t0, t0 + n) of every batch of a host array [batch][len][width]
// to/from a packed device array [batch][n][width].
cudaError_t copy_piece(void* dst, const void* src, bool to_device, int64_t batch, int64_t len, int64_t t0, int64_t n,
                       size_t row_bytes, cudaStream_t st) {
  const size_t piece_pitch = (size_t)n * row_bytes, full_pitch = (size_t)len * row_bytes;
  if (to_device)
    return cudaMemcpy2DAsync(dst, piece_pitch, static_cast<const char*>(src) + (size_t)t0 * row_bytes, full_pitch,
                             piece_pitch, (size_t)batch, cudaMemcpyHostToDevice, st);
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + (size_t)t0 * row_bytes, full_pitch, src, piece_pitch,
                           piece_pitch, (size_t)batch, cudaMemcpyDeviceToHost, st);
}

int scan_host_pipelined(const void* u, const void* delta, const float* A, const void* B, const void* C,
                        const float* D, void* y, float* final_state, int64_t batch, int64_t len, int64_t channels,
                        int64_t nstate, int64_t piece_len, int dtype, cudaStream_t s0) {
  cudaStream_t s1 = nullptr;
  if (int st = aux_stream(&s1)) return st;
  const size_t es = (size_t)elem_size(dtype);
  int64_t P = piece_len > 0 ? piece_len : std::max<int64_t>(256, ((len + 7) / 8 + 63) / 64 * 64);
  P = std::min<int64_t>(P, len);
  const int64_t pieces = (len + P - 1) / P;
  const size_t xb = (size_t)batch * (size_t)P * (size_t)channels * es;  // u, delta or y of one piece
  const size_t bb = (size_t)batch * (size_t)P * (size_t)nstate * es;    // B or C of one piece
  const size_t hb = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
  const size_t ab = sizeof(float) * (size_t)channels * (size_t)(nstate + 1);
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  const size_t per_set = 3 * al(xb) + 2 * al(bb) + al(hb);
  const size_t total = 2 * per_set + al(ab);
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};  // s0 ready for s1, state ready on s0 / s1
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MAMBA_ERR_CUDA;
  int status = MAMBA_OK;
  auto fail = [&](cudaError_t e) {
    if (e != cudaSuccess && status == MAMBA_OK) status = MAMBA_ERR_CUDA;
    return status != MAMBA_OK;
  };
  unsigned char* mem = nullptr;
  if (!fail(scratch_alloc(reinterpret_cast<void**>(&mem), total, s0))) {
    float* dA = reinterpret_cast<float*>(mem + 2 * per_set);
    float* dD = D ? dA + (size_t)channels * nstate : nullptr;
    fail(cudaMemcpyAsync(dA, A, sizeof(float) * (size_t)channels * nstate, cudaMemcpyHostToDevice, s0));
    if (D) fail(cudaMemcpyAsync(dD, D, sizeof(float) * (size_t)channels, cudaMemcpyHostToDevice, s0));
    // s1 starts after everything enqueued on s0 so far (the caller's work, the allocation, A and D)
    fail(cudaEventRecord(ev[0], s0));
    fail(cudaStreamWaitEvent(s1, ev[0], 0));
    float* state_prev = nullptr;
    for (int64_t k = 0; k < pieces && status == MAMBA_OK; ++k) {
      cudaStream_t st = (k & 1) ? s1 : s0;
      unsigned char* set = mem + (size_t)(k & 1) * per_set;
      void* du = set;
      void* ddl = set + al(xb);
      void* dy = set + 2 * al(xb);
      void* dB = set + 3 * al(xb);
      void* dC = set + 3 * al(xb) + al(bb);
      float* dh = reinterpret_cast<float*>(set + 3 * al(xb) + 2 * al(bb));
      const int64_t t0 = k * P, n = std::min<int64_t>(P, len - t0);
      fail(copy_piece(du, u, true, batch, len, t0, n, (size_t)channels * es, st));
      fail(copy_piece(ddl, delta, true, batch, len, t0, n, (size_t)channels * es, st));
      fail(copy_piece(dB, B, true, batch, len, t0, n, (size_t)nstate * es, st));
      fail(copy_piece(dC, C, true, batch, len, t0, n, (size_t)nstate * es, st));
      if (k > 0) fail(cudaStreamWaitEvent(st, ev[1 + ((k - 1) & 1)], 0));  // piece k-1's final state
      if (status != MAMBA_OK) break;
      const int sc = dispatch_nstate(nstate, [&](auto ns) {
        constexpr int NS = decltype(ns)::value;
        return dtype == MAMBA_BF16 ? launch_scan<__nv_bfloat16, NS>(du, ddl, dA, dB, dC, dD, state_prev, dy, dh, batch,
                                                                    n, channels, 0, 0u, dtype, st, false)
                                   : launch_scan<float, NS>(du, ddl, dA, dB, dC, dD, state_prev, dy, dh, batch, n,
                                                            channels, 0, 0u, dtype, st, false);
      });
      if (sc != MAMBA_OK) {
        status = sc;
        break;
      }
      fail(cudaEventRecord(ev[1 + (k & 1)], st));
      fail(copy_piece(y, dy, false, batch, len, t0, n, (size_t)channels * es, st));
      state_prev = dh;
      if (k == pieces - 1 && final_state)
        fail(cudaMemcpyAsync(final_state, dh, hb, cudaMemcpyDeviceToHost, st));
    }
    // join: s0 continues after everything on s1, then the memory goes back
    fail(cudaEventRecord(ev[0], s1));
    fail(cudaStreamWaitEvent(s0, ev[0], 0));
    fail(cudaFreeAsync(mem, s0));
  }
  for (auto& e : ev) cudaEventDestroy(e);
  return status;
}

__global__ void expire_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    // nothing ever arrives on `bar`: the bounded wait must run out
    if (!mbar_wait_bounded(&bar, 0, limit_ns)) record_device_error(MAMBA_ERR_TIMEOUT);
  }
}

// --- Mamba-2's restricted scan (ssd.cuh) ------------------------------------
// Super-chunks per sequence (a CTA's unit): one when the sequences fill at
// least half of the resident CTA slots, else enough for two waves of slots
// (a CTA walks its chunks in order, so parallelism wins for long sequences;
// each super-chunk after the first adds a correction walk of a few chunks).
int64_t ssd_supers(int64_t seqs, int64_t chunks, int64_t slots, int64_t requested) {
  int64_t s = requested > 0 ? requested
                            : (seqs * 2 >= slots ? 1 : std::max<int64_t>(1, (2 * slots + seqs - 1) / seqs));
  return std::max<int64_t>(1, std::min(s, chunks));
}

template <int N>
int launch_ssd(SsdArgs a, int64_t batch, int64_t supers_req, cudaStream_t stream) {
  using L = SsdSmem<N>;
  auto main_k = ssd_chunk_kernel<N>;
  if (cudaFuncSetAttribute(main_k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  int sms = 0, per_sm = 0;
  if (current_sms(&sms) != MAMBA_OK) return MAMBA_ERR_CUDA;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, main_k, kSsdThreads, L::kBytes) != cudaSuccess ||
      per_sm < 1)
    return MAMBA_ERR_CUDA;
  // tensor memory: kSsdTmemCols columns per CTA out of 512 per SM
  per_sm = std::min(per_sm, 512 / kSsdTmemCols);
  a.wait_limit_ns = kWaitLimitNs;
  const int64_t seqs = batch * a.heads;  // one CTA per (batch row, head, super-chunk)
  const int64_t chunks = (a.len + kSsdQ - 1) / kSsdQ;
  int64_t S = ssd_supers(seqs, chunks, (int64_t)sms * per_sm, supers_req);
  const int64_t per = (chunks + S - 1) / S;
  S = (chunks + per - 1) / per;
  a.super_len = per * kSsdQ;
  a.supers = (int)S;
  if (seqs * S >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  unsigned char* mem = nullptr;
  if (S > 1) {  // every super-chunk's end state from zero and its decay
    const size_t n_agg = (size_t)seqs * (size_t)S;
    const size_t st_bytes = n_agg * kSsdP * N * sizeof(float);
    if (scratch_alloc(reinterpret_cast<void**>(&mem), st_bytes + n_agg * sizeof(float), stream) != cudaSuccess)
      return MAMBA_ERR_CUDA;
    a.agg_state = reinterpret_cast<float*>(mem);
    a.agg_decay = reinterpret_cast<float*>(mem + st_bytes);
  }
  // x, B and C tiles by TMA when the maps can be made (else cp.async)
  CUtensorMap mx, mb, mc;
  std::memset(&mx, 0, sizeof(mx));
  std::memset(&mb, 0, sizeof(mb));
  std::memset(&mc, 0, sizeof(mc));
  const uint64_t channels = (uint64_t)a.heads * kSsdP;
  a.tma = (make_map_core_tiles(&mx, a.x, channels, (uint64_t)a.len, (uint64_t)batch, 8) &&
           make_map_core_tiles(&mb, a.B, N, (uint64_t)a.len, (uint64_t)batch, N / 8) &&
           make_map_core_tiles(&mc, a.C, N, (uint64_t)a.len, (uint64_t)batch, N / 8))
              ? 1
              : 0;
  int st = MAMBA_OK;
  if (launch_pdl(main_k, dim3((unsigned)(seqs * S)), dim3(kSsdThreads), L::kBytes, stream, a, mx, mb, mc) !=
      cudaSuccess)
    st = MAMBA_ERR_CUDA;
  // the states entering super-chunks 1..S-1, their effect on y, the final state
  if (st == MAMBA_OK && S > 1 &&
      launch_pdl(ssd_fix_kernel<N>, dim3((unsigned)(seqs * (S - 1))), dim3(128), 0, stream, a) != cudaSuccess)
    st = MAMBA_ERR_CUDA;
  if (mem && cudaFreeAsync(mem, stream) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

// --- complex-valued state (complex_scan.cuh) ---------------------------------
template <typename TIO, int N>
int launch_complex(ComplexArgs a, int64_t batch, int64_t supers_req, cudaStream_t stream) {
  using L = ComplexSmem<TIO, N>;
  constexpr int kES = (int)sizeof(TIO);
  a.groups = (int)((a.channels + L::kCPW - 1) / L::kCPW);
  a.async = ((int64_t)a.channels * kES) % 16 == 0 && (N * kES) % 16 == 0 && aligned(a.u, 16) &&
            aligned(a.delta, 16) && aligned(a.y, 16) && aligned(a.B, 16) && aligned(a.C, 16);
  auto main_k = complex_scan_kernel<TIO, N, false>;
  auto agg_k = complex_scan_kernel<TIO, N, true>;
  if (cudaFuncSetAttribute(main_k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess ||
      cudaFuncSetAttribute(agg_k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  int sms = 0, per_sm = 0;
  if (current_sms(&sms) != MAMBA_OK) return MAMBA_ERR_CUDA;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, main_k, kCplxWarps * 32, L::kBytes) != cudaSuccess ||
      per_sm < 1)
    return MAMBA_ERR_CUDA;
  const int64_t seqs = batch * a.groups;  // one warp each
  const int64_t blocks = (a.len + kCplxBlock - 1) / kCplxBlock;
  // one super-chunk per sequence when the warps fill at least half of the
  // slots, else as many as fit the slots in one wave (the aggregate pass
  // costs nearly a full pass here: its exponentials dominate)
  const int64_t slots = (int64_t)sms * per_sm * kCplxWarps;
  int64_t S = supers_req > 0 ? supers_req : (seqs * 2 >= slots ? 1 : std::max<int64_t>(1, slots / seqs));
  S = std::max<int64_t>(1, std::min(S, blocks));
  const int64_t per = (blocks + S - 1) / S;
  S = (blocks + per - 1) / per;
  a.super_len = per * kCplxBlock;
  a.supers = (int)S;
  if (seqs * S >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  unsigned char* mem = nullptr;
  if (S > 1) {
    const size_t slots = (size_t)batch * (size_t)(S - 1) * (size_t)a.channels;
    const size_t h_bytes = (slots * N * 2 * sizeof(float) + 15) / 16 * 16;
    if (scratch_alloc(reinterpret_cast<void**>(&mem), h_bytes + slots * sizeof(double), stream) != cudaSuccess)
      return MAMBA_ERR_CUDA;
    a.agg_h = reinterpret_cast<float*>(mem);
    a.agg_sd = reinterpret_cast<double*>(mem + h_bytes);
    a.jobs = seqs * (S - 1);
    if (launch_pdl(agg_k, dim3((unsigned)((a.jobs + kCplxWarps - 1) / kCplxWarps)), dim3(kCplxWarps * 32), L::kBytes,
                   stream, a) != cudaSuccess) {
      cudaFreeAsync(mem, stream);
      return MAMBA_ERR_CUDA;
    }
  }
  a.jobs = seqs * S;
  int st = MAMBA_OK;
  if (launch_pdl(main_k, dim3((unsigned)((a.jobs + kCplxWarps - 1) / kCplxWarps)), dim3(kCplxWarps * 32), L::kBytes,
                 stream, a) != cudaSuccess)
    st = MAMBA_ERR_CUDA;
  if (mem && cudaFreeAsync(mem, stream) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

}  // namespace
}  // namespace mamba

using namespace mamba;

extern "C" {

const char* mamba_status_string(int status) {
  switch (status) {
    case MAMBA_OK: return "ok";
    case MAMBA_ERR_INVALID_ARG: return "invalid argument";
    case MAMBA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MAMBA_ERR_CUDA: return "CUDA error";
    case MAMBA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int mamba_scan_supported_nstate(int64_t nstate) {
  return (nstate == 4 || nstate == 8 || nstate == 16 || nstate == 32) ? 1 : 0;
}

int mamba_scan_plan(int64_t batch, int64_t len, int64_t channels, int64_t nstate, int64_t chunk_len, int dtype,
                    int sm_count, mamba_scan_plan_t* out) {
  if (!out || (dtype != MAMBA_F32 && dtype != MAMBA_BF16)) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || chunk_len < 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_scan_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  std::memset(out, 0, sizeof(*out));
  if (batch == 0 || channels == 0 || len == 0) return MAMBA_OK;  // nothing is launched
  int sms = sm_count;
  if (sms <= 0) {
    if (int st = current_sms(&sms)) return st;
  }
  const Plan pl = choose_plan(batch, len, channels, nstate, sms, dtype, chunk_len, true);
  out->supers = pl.supers;
  out->super_len = pl.super_len;
  out->chunk_len = pl.chunk_len;
  out->jobs = full_jobs(pl);
  out->kernels = kernels_per_call(pl);
  out->scratch_bytes =
      (int64_t)scratch_layout(pl, (int)nstate, batch, len, tile_for(dtype, pl.cw), dtype == MAMBA_BF16).total;
  out->ctas = std::min<int64_t>(sms, (out->jobs + pl.cw - 1) / pl.cw);
  out->consumer_warps = pl.cw;
  return MAMBA_OK;
}

int mamba_selective_scan_ex(const void* u, const void* delta, const float* A, const void* B, const void* C,
                            const float* D, const float* initial_state, void* y, float* final_state,
                            int64_t batch, int64_t len, int64_t channels, int64_t nstate, int64_t chunk_len,
                            unsigned flags, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || chunk_len < 0) return MAMBA_ERR_INVALID_ARG;
  if (flags & ~(MAMBA_SCAN_GENERAL_A | MAMBA_SCAN_EULER | MAMBA_SCAN_TRAPEZOID)) return MAMBA_ERR_INVALID_ARG;
  if ((flags & MAMBA_SCAN_EULER) && (flags & MAMBA_SCAN_TRAPEZOID)) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_scan_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  const size_t es = (size_t)elem_size(dtype);
  if (len > 0) {
    if (!u || !delta || !B || !C || !y || !A) return MAMBA_ERR_INVALID_ARG;
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) || !aligned(y, es))
      return MAMBA_ERR_INVALID_ARG;
  }
  if ((A && !aligned(A, 4)) || (D && !aligned(D, 4)) || (final_state && !aligned(final_state, 4)) ||
      (initial_state && !aligned(initial_state, 4)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;

  cudaGetLastError();  // clear a stale, non-sticky error so the status below is ours
  const size_t state_bytes = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    cudaError_t e = initial_state
                        ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(final_state, 0, state_bytes, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  return dispatch_nstate(nstate, [&](auto ns) {
    constexpr int NS = decltype(ns)::value;
    if (dtype == MAMBA_BF16)
      return launch_scan<__nv_bfloat16, NS>(u, delta, A, B, C, D, initial_state, y, final_state, batch, len, channels,
                                            chunk_len, flags, dtype, stream, false);
    return launch_scan<float, NS>(u, delta, A, B, C, D, initial_state, y, final_state, batch, len, channels,
                                  chunk_len, flags, dtype, stream, false);
  });
}

int mamba_mimo_supported(int64_t ranks, int64_t nstate) {
  return ((ranks == 2 || ranks == 4) && nstate == 16) ? 1 : 0;
}

int mamba_selective_scan_mimo(const void* u, const void* delta, const float* A, const void* B, const void* C,
                              const float* D, const float* initial_state, void* y, float* final_state,
                              int64_t batch, int64_t len, int64_t ranks, int64_t channels, int64_t nstate,
                              unsigned flags, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || ranks <= 0) return MAMBA_ERR_INVALID_ARG;
  if (flags & ~MAMBA_SCAN_GENERAL_A) {
    if (flags & ~(MAMBA_SCAN_GENERAL_A | MAMBA_SCAN_EULER | MAMBA_SCAN_TRAPEZOID)) return MAMBA_ERR_INVALID_ARG;
    return MAMBA_ERR_UNSUPPORTED;  // zero-order hold only
  }
  if (!mamba_mimo_supported(ranks, nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  const size_t es = (size_t)elem_size(dtype);
  if (len > 0) {
    if (!u || !delta || !B || !C || !y || !A) return MAMBA_ERR_INVALID_ARG;
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) || !aligned(y, es))
      return MAMBA_ERR_INVALID_ARG;
  }
  if ((A && !aligned(A, 4)) || (D && !aligned(D, 4)) || (final_state && !aligned(final_state, 4)) ||
      (initial_state && !aligned(initial_state, 4)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len * ranks >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;

  cudaGetLastError();  // clear a stale, non-sticky error so the status below is ours
  const size_t state_bytes = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    cudaError_t e = initial_state
                        ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(final_state, 0, state_bytes, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  auto go = [&](auto rk) {
    constexpr int R = decltype(rk)::value;
    if (dtype == MAMBA_BF16)
      return launch_scan_mimo<__nv_bfloat16, 16, R>(u, delta, A, B, C, D, initial_state, y, final_state, batch, len,
                                                    channels, flags, dtype, stream);
    return launch_scan_mimo<float, 16, R>(u, delta, A, B, C, D, initial_state, y, final_state, batch, len, channels,
                                          flags, dtype, stream);
  };
  return ranks == 2 ? go(std::integral_constant<int, 2>{}) : go(std::integral_constant<int, 4>{});
}

int mamba_selective_scan(const void* u, const void* delta, const float* A, const void* B, const void* C,
                         const float* D, void* y, float* final_state, int64_t batch, int64_t len, int64_t channels,
                         int64_t nstate, int dtype, mamba_stream_t stream) {
  return mamba_selective_scan_ex(u, delta, A, B, C, D, nullptr, y, final_state, batch, len, channels, nstate, 0, 0u,
                                 dtype, stream);
}

int mamba_selective_scan_host(const void* u, const void* delta, const float* A, const void* B, const void* C,
                              const float* D, void* y, float* final_state, int64_t batch, int64_t len,
                              int64_t channels, int64_t nstate, int64_t piece_len, int dtype,
                              mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || piece_len < 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_scan_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  if (!A) return MAMBA_ERR_INVALID_ARG;
  if (len > 0 && (!u || !delta || !B || !C || !y)) return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  cudaGetLastError();
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    const size_t hb = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
    std::memset(final_state, 0, hb);  // h_0 = 0 and no token: the final state is zero
    return MAMBA_OK;
  }
  return scan_host_pipelined(u, delta, A, B, C, D, y, final_state, batch, len, channels, nstate, piece_len, dtype,
                             stream);
}

int mamba_selective_scan_backward(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                  const float* D, const float* initial_state, const void* dy,
                                  const float* d_final_state, void* du, void* ddelta, float* dA, float* dB,
                                  float* dC, float* dD, float* d_initial_state, int64_t batch, int64_t len,
                                  int64_t channels, int64_t nstate, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0) return MAMBA_ERR_INVALID_ARG;
  if (nstate != 4 && nstate != 8 && nstate != 16) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  if (!A || !dA || !dB || !dC || (D && !dD)) return MAMBA_ERR_INVALID_ARG;
  const size_t es = (size_t)elem_size(dtype);
  if (len > 0) {
    if (!u || !delta || !B || !C || !dy || !du || !ddelta) return MAMBA_ERR_INVALID_ARG;
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) || !aligned(dy, es) ||
        !aligned(du, es) || !aligned(ddelta, es))
      return MAMBA_ERR_INVALID_ARG;
  }
  if (!aligned(A, 4) || !aligned(dA, 4) || !aligned(dB, 4) || !aligned(dC, 4) || (D && !aligned(D, 4)) ||
      (dD && !aligned(dD, 4)) || (initial_state && !aligned(initial_state, 4)) ||
      (d_final_state && !aligned(d_final_state, 4)) || (d_initial_state && !aligned(d_initial_state, 4)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  cudaGetLastError();
  const size_t state_bytes = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
  // gradients that are sums start at zero
  if (cudaMemsetAsync(dA, 0, sizeof(float) * (size_t)channels * (size_t)nstate, stream) != cudaSuccess ||
      cudaMemsetAsync(dB, 0, sizeof(float) * (size_t)batch * (size_t)len * (size_t)nstate, stream) != cudaSuccess ||
      cudaMemsetAsync(dC, 0, sizeof(float) * (size_t)batch * (size_t)len * (size_t)nstate, stream) != cudaSuccess ||
      (dD && D && cudaMemsetAsync(dD, 0, sizeof(float) * (size_t)channels, stream) != cudaSuccess))
    return MAMBA_ERR_CUDA;
  if (len == 0) {
    if (!d_initial_state) return MAMBA_OK;
    const cudaError_t e = d_final_state ? cudaMemcpyAsync(d_initial_state, d_final_state, state_bytes,
                                                          cudaMemcpyDeviceToDevice, stream)
                                        : cudaMemsetAsync(d_initial_state, 0, state_bytes, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  int sms = 0;
  if (int st = current_sms(&sms)) return st;
  return dispatch_nstate(nstate, [&](auto ns) -> int {
    constexpr int NS = decltype(ns)::value;
    if constexpr (NS > 16) {
      return MAMBA_ERR_UNSUPPORTED;
    } else {
      auto run = [&](auto tio) -> int {
        using TIO = decltype(tio);
        constexpr int T = ScanCfg<TIO, NS>::kTile;
        const int64_t ntiles = (len + T - 1) / T;
        const int64_t groups_d = (channels + 31) / 32;
        const int64_t streams = batch * groups_d;
        // The sequence is cut into S super-chunks run in parallel; their
        // incoming adjoints come from the reverse aggregates of the later
        // super-chunks.  The S * streams work items are dealt to the resident
        // warps in rounds, each item 1/S of a sequence: the reverse pass
        // takes about ceil(S streams / resident) / S of one warp's walk over a
        // whole sequence, and the aggregate pass adds about kBwdAggCost of
        // that per (S-1)/S.  S minimises the sum (measured on 8 x 2048 x 3072:
        // S = 4 -> 3, 2.574 -> 2.373 ms; on 4 x 8192 x 5120: S = 4 -> 11,
        // 8.38 -> 7.50 ms).
        const int64_t resident = kBwdCtasPerSm * (int64_t)sms * kBwdWarps;
        constexpr double kBwdAggCost = 0.2;
        int64_t S = 1;
        {
          double best = 1e30;
          for (int64_t s = 1; s <= std::min<int64_t>(ntiles, 64); ++s) {
            const double rounds = (double)((s * streams + resident - 1) / resident);
            const double cost = rounds / (double)s + kBwdAggCost * (double)(s - 1) / (double)s;
            if (cost < best - 1e-9) {
              best = cost;
              S = s;
            }
          }
        }
        const int64_t super_tiles = (ntiles + S - 1) / S;
        const int64_t supers = (ntiles + super_tiles - 1) / super_tiles;
        const int64_t items = supers * streams;
        const int64_t ctas = std::min<int64_t>((items + kBwdWarps - 1) / kBwdWarps, kBwdCtasPerSm * (int64_t)sms);
        auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
        const size_t ck_bytes = al(sizeof(float) * (size_t)batch * (size_t)ntiles * (size_t)channels * NS);
        const size_t sc_bytes = al(sizeof(float) * (size_t)ctas * kBwdWarps * (T / 2 + 1) * 32 * NS);
        const size_t mu_bytes = al(sizeof(float) * (size_t)supers * (size_t)streams * 32 * NS);
        const size_t sd_bytes = al(sizeof(float) * (size_t)supers * (size_t)streams * 32);
        // bf16 B and C are widened to fp32 once (fp32 B and C are read in place)
        constexpr bool kWiden = sizeof(TIO) == 2;
        const size_t row_elems = (size_t)batch * (size_t)len * NS;
        const size_t wd_bytes = kWiden ? al(sizeof(float) * row_elems) : 0;
        unsigned char* mem = nullptr;
        if (scratch_alloc(reinterpret_cast<void**>(&mem), ck_bytes + sc_bytes + mu_bytes + sd_bytes + 2 * wd_bytes,
                          stream) != cudaSuccess)
          return MAMBA_ERR_CUDA;
        float* ckpt = reinterpret_cast<float*>(mem);
        unsigned char* wd = mem + ck_bytes + sc_bytes + mu_bytes + sd_bytes;
        const float* Bf = kWiden ? reinterpret_cast<const float*>(wd) : static_cast<const float*>(B);
        const float* Cf = kWiden ? reinterpret_cast<const float*>(wd + wd_bytes) : static_cast<const float*>(C);
        int st = MAMBA_OK;
        if constexpr (kWiden) {
          const int vec = (aligned(B, 16) && aligned(C, 16) && row_elems % 8 == 0) ? 1 : 0;
          const int64_t work = vec ? (int64_t)(row_elems / 8) : (int64_t)row_elems;
          const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 8 * sms));
          if (launch_pdl(bwd_widen_kernel, dim3(blocks), dim3(256), 0, stream,
                         static_cast<const __nv_bfloat16*>(B), static_cast<const __nv_bfloat16*>(C),
                         const_cast<float*>(Bf), const_cast<float*>(Cf), (int64_t)row_elems, vec) != cudaSuccess)
            st = MAMBA_ERR_CUDA;
        }
        // forward pass that only leaves the state before every tile
        if (st == MAMBA_OK)
          st = launch_scan<TIO, NS>(u, delta, A, B, C, D, initial_state, nullptr, nullptr, batch, len, channels, 0,
                                    0u, dtype, stream, false, ckpt);
        if (st == MAMBA_OK) {
          BwdArgs<TIO> a{static_cast<const TIO*>(u), static_cast<const TIO*>(delta), A, Bf, Cf, D,
                         static_cast<const TIO*>(dy), d_final_state, ckpt, reinterpret_cast<float*>(mem + ck_bytes),
                         static_cast<TIO*>(du), static_cast<TIO*>(ddelta), dA, dB, dC, D ? dD : nullptr,
                         d_initial_state, batch, len, channels, (int)groups_d, T,
                         (aligned(Bf, 16) && aligned(Cf, 16)) ? 1 : 0, (int)supers, (int)super_tiles,
                         reinterpret_cast<float*>(mem + ck_bytes + sc_bytes),
                         reinterpret_cast<float*>(mem + ck_bytes + sc_bytes + mu_bytes), 0};
          // tiles staged in shared memory when every row piece is a whole,
          // aligned 16-byte copy
          a.staged = ((channels * (int64_t)es) % 16 == 0 && aligned(u, 16) && aligned(delta, 16) &&
                      aligned(dy, 16) && aligned(Bf, 16) && aligned(Cf, 16))
                         ? 1
                         : 0;
          if (supers > 1) {
            const int64_t agg_items = (supers - 1) * streams;
            const int agg_smem = a.staged ? kBwdWarps * bwd_agg_stage_bytes<TIO, NS>(T) : 0;
            if (agg_smem > 0 && cudaFuncSetAttribute(scan_backward_aggregate_kernel<TIO, NS>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     agg_smem) != cudaSuccess)
              st = MAMBA_ERR_CUDA;
            if (st == MAMBA_OK &&
                launch_pdl(scan_backward_aggregate_kernel<TIO, NS>,
                           dim3((unsigned)((agg_items + kBwdWarps - 1) / kBwdWarps)), dim3(kBwdWarps * 32),
                           (size_t)agg_smem, stream, a) != cudaSuccess)
              st = MAMBA_ERR_CUDA;
          }
          const int smem = kBwdWarps * bwd_warp_smem<TIO, NS>(T, a.staged != 0);
          if (st == MAMBA_OK &&
              cudaFuncSetAttribute(scan_backward_kernel<TIO, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   smem) != cudaSuccess)
            st = MAMBA_ERR_CUDA;
          if (st == MAMBA_OK &&
              launch_pdl(scan_backward_kernel<TIO, NS>, dim3((unsigned)ctas), dim3(kBwdWarps * 32), (size_t)smem,
                         stream, a) != cudaSuccess)
            st = MAMBA_ERR_CUDA;
        }
        if (cudaFreeAsync(mem, stream) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
        return st;
      };
      return dtype == MAMBA_BF16 ? run(__nv_bfloat16{}) : run(float{});
    }
  });
}

int mamba_selective_scan_noalloc(const void* u, const void* delta, const float* A, const void* B, const void* C,
                                 const float* D, void* y, float* final_state, int64_t batch, int64_t len,
                                 int64_t channels, int64_t nstate, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_scan_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  const size_t es = (size_t)elem_size(dtype);
  if (len > 0) {
    if (!u || !delta || !B || !C || !y || !A) return MAMBA_ERR_INVALID_ARG;
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) || !aligned(y, es))
      return MAMBA_ERR_INVALID_ARG;
  }
  if ((A && !aligned(A, 4)) || (D && !aligned(D, 4)) || (final_state && !aligned(final_state, 4)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  cudaGetLastError();
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    const size_t state_bytes = sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
    return cudaMemsetAsync(final_state, 0, state_bytes, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  return dispatch_nstate(nstate, [&](auto ns) {
    constexpr int NS = decltype(ns)::value;
    if (dtype == MAMBA_BF16)
      return launch_scan<__nv_bfloat16, NS>(u, delta, A, B, C, D, nullptr, y, final_state, batch, len, channels, 0,
                                            0u, dtype, stream, true);
    return launch_scan<float, NS>(u, delta, A, B, C, D, nullptr, y, final_state, batch, len, channels, 0, 0u, dtype,
                                  stream, true);
  });
}

int mamba_state_update(float* state, const void* x, const void* delta, const float* A, const void* B, const void* C,
                       const float* D, void* y, int64_t batch, int64_t channels, int64_t nstate, int dtype,
                       mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || channels < 0 || nstate <= 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_scan_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  if (!state || !x || !delta || !A || !B || !C || !y) return MAMBA_ERR_INVALID_ARG;
  const size_t es = (size_t)elem_size(dtype);
  if (!aligned(state, 16) || !aligned(A, 16) || (D && !aligned(D, 4)) || !aligned(x, es) || !aligned(delta, es) ||
      !aligned(y, es) || !aligned(B, 4 * es) || !aligned(C, 4 * es))
    return MAMBA_ERR_INVALID_ARG;
  cudaGetLastError();
  constexpr int kRows = 4;  // batch rows per thread
  // programmatic launch: a step's setup overlaps the end of the previous
  // kernel of the stream (the kernel waits for it before touching memory)
  return dispatch_nstate(nstate, [&](auto ns) {
    constexpr int NS = decltype(ns)::value;
    constexpr int kChanPerCta = kDecodeWarps * (32 / (NS / 4));  // NS/4 lanes per (batch, channel) row
    const int64_t gx = (channels + kChanPerCta - 1) / kChanPerCta;
    const int64_t gy = (batch + kRows - 1) / kRows;
    if (gy > 65535 || gx > 0x7fffffff) return (int)MAMBA_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)gx, (unsigned)gy);
    cudaError_t err;
    if (dtype == MAMBA_BF16) {
      DecodeArgs<__nv_bfloat16, NS> a{state, static_cast<const __nv_bfloat16*>(x),
                                      static_cast<const __nv_bfloat16*>(delta), A,
                                      static_cast<const __nv_bfloat16*>(B), static_cast<const __nv_bfloat16*>(C), D,
                                      static_cast<__nv_bfloat16*>(y), batch, channels};
      err = launch_pdl(state_update_kernel<__nv_bfloat16, NS, kRows, true>, grid, dim3(kDecodeWarps * 32), 0, stream,
                       a);
    } else {
      DecodeArgs<float, NS> a{state, static_cast<const float*>(x), static_cast<const float*>(delta), A,
                              static_cast<const float*>(B), static_cast<const float*>(C), D,
                              static_cast<float*>(y), batch, channels};
      err = launch_pdl(state_update_kernel<float, NS, kRows, false>, grid, dim3(kDecodeWarps * 32), 0, stream, a);
    }
    return err == cudaSuccess ? (int)MAMBA_OK : (int)MAMBA_ERR_CUDA;
  });
}

int mamba_state_update_mimo(float* state, const void* x, const void* delta, const float* A, const void* B,
                            const void* C, const float* D, void* y, int64_t batch, int64_t ranks, int64_t channels,
                            int64_t nstate, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || channels < 0 || nstate <= 0 || ranks <= 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_mimo_supported(ranks, nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  if (!state || !x || !delta || !A || !B || !C || !y) return MAMBA_ERR_INVALID_ARG;
  const size_t es = (size_t)elem_size(dtype);
  if (!aligned(state, 16) || !aligned(A, 16) || (D && !aligned(D, 4)) || !aligned(x, es) || !aligned(delta, es) ||
      !aligned(y, es) || !aligned(B, 4 * es) || !aligned(C, 4 * es))
    return MAMBA_ERR_INVALID_ARG;
  cudaGetLastError();
  constexpr int NS = 16;
  // batch rows per thread: one keeps the registers low enough for more
  // resident warps, which the step needs to keep loads in flight (256 x 5120
  // rows, 4 inputs and outputs: 68 us with one row, 77 with two, 103 with four)
#ifndef MAMBA_MIMO_DECODE_ROWS
#define MAMBA_MIMO_DECODE_ROWS 1
#endif
  constexpr int kRows = MAMBA_MIMO_DECODE_ROWS;
  constexpr int kChanPerCta = kDecodeWarps * (32 / (NS / 4));
  const int64_t gx = (channels + kChanPerCta - 1) / kChanPerCta;
  const int64_t gy = (batch + kRows - 1) / kRows;
  if (gy > 65535 || gx > 0x7fffffff) return MAMBA_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)gx, (unsigned)gy);
  auto go = [&](auto rk) {
    constexpr int R = decltype(rk)::value;
    cudaError_t err;
    if (dtype == MAMBA_BF16) {
      DecodeArgs<__nv_bfloat16, NS> a{state, static_cast<const __nv_bfloat16*>(x),
                                      static_cast<const __nv_bfloat16*>(delta), A,
                                      static_cast<const __nv_bfloat16*>(B), static_cast<const __nv_bfloat16*>(C), D,
                                      static_cast<__nv_bfloat16*>(y), batch, channels};
      err = launch_pdl(state_update_mimo_kernel<__nv_bfloat16, NS, R, kRows, true>, grid, dim3(kDecodeWarps * 32), 0,
                       stream, a);
    } else {
      DecodeArgs<float, NS> a{state, static_cast<const float*>(x), static_cast<const float*>(delta), A,
                              static_cast<const float*>(B), static_cast<const float*>(C), D,
                              static_cast<float*>(y), batch, channels};
      err = launch_pdl(state_update_mimo_kernel<float, NS, R, kRows, false>, grid, dim3(kDecodeWarps * 32), 0, stream,
                       a);
    }
    return err == cudaSuccess ? (int)MAMBA_OK : (int)MAMBA_ERR_CUDA;
  };
  return ranks == 2 ? go(std::integral_constant<int, 2>{}) : go(std::integral_constant<int, 4>{});
}

int mamba_ssd_supported_nstate(int64_t nstate) { return nstate == 16 || nstate == 32 || nstate == 64; }

int mamba_ssd_scan(const void* x, const void* dt, const float* A, const void* B, const void* C, const float* D,
                   const float* initial_state, void* y, float* final_state, int64_t batch, int64_t len,
                   int64_t heads, int64_t headdim, int64_t nstate, int64_t supers, unsigned flags, int dtype,
                   mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || heads < 0 || headdim <= 0 || nstate <= 0 || supers < 0) return MAMBA_ERR_INVALID_ARG;
  if (flags & ~(MAMBA_SCAN_GENERAL_A | MAMBA_SCAN_EULER | MAMBA_SCAN_TRAPEZOID)) return MAMBA_ERR_INVALID_ARG;
  if ((flags & MAMBA_SCAN_EULER) && (flags & MAMBA_SCAN_TRAPEZOID)) return MAMBA_ERR_INVALID_ARG;
  if (flags & MAMBA_SCAN_TRAPEZOID) return MAMBA_ERR_UNSUPPORTED;
  if (dtype != MAMBA_BF16 || headdim != kSsdP || !mamba_ssd_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0) return MAMBA_OK;
  if (len > 0) {
    if (!x || !dt || !A || !B || !C || !y) return MAMBA_ERR_INVALID_ARG;
    // x, B, C and y move in 16-byte pieces; dt in 2-byte ones
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) || !aligned(dt, 2))
      return MAMBA_ERR_INVALID_ARG;
  }
  if ((A && !aligned(A, 4)) || (D && !aligned(D, 8)) || (final_state && !aligned(final_state, 4)) ||
      (initial_state && !aligned(initial_state, 4)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || heads * headdim >= (int64_t(1) << 31) || batch * heads >= (int64_t(1) << 31))
    return MAMBA_ERR_UNSUPPORTED;

  cudaGetLastError();  // clear a stale, non-sticky error so the status below is ours
  const size_t state_bytes = sizeof(float) * (size_t)batch * (size_t)(heads * headdim) * (size_t)nstate;
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    cudaError_t e = initial_state
                        ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(final_state, 0, state_bytes, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  SsdArgs a = {};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.dt = static_cast<const __nv_bfloat16*>(dt);
  a.A = A;
  a.B = static_cast<const __nv_bfloat16*>(B);
  a.C = static_cast<const __nv_bfloat16*>(C);
  a.D = D;
  a.h0 = initial_state;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.final_state = final_state;
  a.len = len;
  a.heads = (int)heads;
  a.euler = (flags & MAMBA_SCAN_EULER) ? 1 : 0;
  switch (nstate) {
    case 16: return launch_ssd<16>(a, batch, supers, stream);
    case 32: return launch_ssd<32>(a, batch, supers, stream);
    default: return launch_ssd<64>(a, batch, supers, stream);
  }
}

int mamba_complex_supported_nstate(int64_t nstate) { return nstate == 4 || nstate == 8 || nstate == 16; }

int mamba_selective_scan_complex(const void* u, const void* delta, const float* A_re, const float* A_im,
                                 const void* B, const void* C, const float* D, const float* initial_state, void* y,
                                 float* final_state, int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                                 int64_t supers, int dtype, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (dtype != MAMBA_F32 && dtype != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || supers < 0) return MAMBA_ERR_INVALID_ARG;
  if (!mamba_complex_supported_nstate(nstate)) return MAMBA_ERR_UNSUPPORTED;
  if (batch == 0 || channels == 0) return MAMBA_OK;
  const size_t es = (size_t)elem_size(dtype);
  if (!A_re || !A_im) return MAMBA_ERR_INVALID_ARG;
  if (len > 0) {
    if (!u || !delta || !B || !C || !y) return MAMBA_ERR_INVALID_ARG;
    if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) || !aligned(y, es))
      return MAMBA_ERR_INVALID_ARG;
  }
  if (!aligned(A_re, 4) || !aligned(A_im, 4) || (D && !aligned(D, 4)) || (final_state && !aligned(final_state, 8)) ||
      (initial_state && !aligned(initial_state, 8)))
    return MAMBA_ERR_INVALID_ARG;
  if (batch * len >= (int64_t(1) << 31) || channels >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;

  cudaGetLastError();  // clear a stale, non-sticky error so the status below is ours
  const size_t state_bytes = 2 * sizeof(float) * (size_t)batch * (size_t)channels * (size_t)nstate;
  if (len == 0) {
    if (!final_state) return MAMBA_OK;
    cudaError_t e = initial_state
                        ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(final_state, 0, state_bytes, stream);
    return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
  }
  ComplexArgs a = {};
  a.u = u;
  a.delta = delta;
  a.A_re = A_re;
  a.A_im = A_im;
  a.B = B;
  a.C = C;
  a.D = D;
  a.h0 = initial_state;
  a.y = y;
  a.final_state = final_state;
  a.len = len;
  a.channels = (int)channels;
  auto go = [&](auto ns) {
    constexpr int NS = decltype(ns)::value;
    return dtype == MAMBA_BF16 ? launch_complex<__nv_bfloat16, NS>(a, batch, supers, stream)
                               : launch_complex<float, NS>(a, batch, supers, stream);
  };
  switch (nstate) {
    case 4: return go(std::integral_constant<int, 4>{});
    case 8: return go(std::integral_constant<int, 8>{});
    default: return go(std::integral_constant<int, 16>{});
  }
}

int mamba_get_device_error(mamba_stream_t stream_, int clear) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // the read (and the clear) are ordered after the work already on `stream`;
  // only that stream is waited for
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  if (clear) {
    static const int kZero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_error, &kZero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
      return MAMBA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MAMBA_ERR_CUDA;
  return v;
}

int64_t mamba_debug_scratch_allocations(void) { return g_scratch_allocs.load(); }

int mamba_trim_scratch_pool(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAMBA_ERR_CUDA;
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_pool_mu);
    pool = g_pool[dev];
  }
  if (pool && cudaMemPoolTrimTo(pool, 0) != cudaSuccess) return MAMBA_ERR_CUDA;
  return MAMBA_OK;
}

int mamba_debug_expire_wait(int64_t limit_ns, mamba_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t lim = std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 1000000000);
  cudaGetLastError();
  expire_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)lim);
  return cudaGetLastError() == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

}  // extern "C"
