/*
 * mamba_ssm.h -- C ABI of the B200 (sm_100a) selective-scan library.
 *
 * The library computes the hot path of the Mamba selective state-space model
 * described on the web page "Mamba SSM Nedir? Transformer Alternatifi Rehberi
 * (2026)":
 *   - section "State Space Model Temelleri": continuous system
 *       h'(t) = A h(t) + B x(t),  y(t) = C h(t) + D x(t);
 *   - section "Ayrık Zamana Geçiş": zero-order-hold discretisation
 *       Abar = exp(Delta A),  Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B,
 *     and the recurrence h_t = Abar h_{t-1} + Bbar x_t,  y_t = C h_t;
 *   - section "Mamba'nın Yeniliği: Selective SSM": B_t, C_t and Delta_t are
 *     given per token (the projections that produce them are not part of
 *     this library);
 *   - section "Paralel Tarama Algoritması": the recurrence is evaluated with a
 *     chunked scan whose chunk results are combined associatively.
 *
 * A is diagonal and real: one value A[d][n] per (channel, state), expected
 * negative (the stability condition of the same page's "Sınırlılıklar ve Açık
 * Sorular" section; not checked).  Each output is y_t = C_t . h_t + D_d x_t
 * with h_t the state after the update at token t.
 *
 * Conventions for every entry point
 *   - Pointers named device memory must be CUDA device (or managed) memory of
 *     the current device, owned by the caller; the library never frees them.
 *   - Layouts are dense row-major with the last index fastest:
 *       u, delta, y            [batch][len][channels]
 *       B, C                   [batch][len][nstate]   (shared by all channels)
 *       A                      [channels][nstate]     float32
 *       D                      [channels]             float32
 *       states                 [batch][channels][nstate] float32
 *   - `dtype` (mamba_dtype_t) is the element type of u, delta, B, C and y
 *     (x, delta, B, C, y for the state update).  A, D and states are float32.
 *     All arithmetic is float32; y is rounded to `dtype` (round to nearest even).
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream): they
 *     validate arguments on the host, enqueue kernels and return.  They never
 *     synchronise.
 *   - Return value: a mamba_status_t.  Argument errors are reported before
 *     anything is enqueued.  A kernel-launch failure returns MAMBA_ERR_CUDA.
 *     A bounded device-side wait that ran out records MAMBA_ERR_TIMEOUT in a
 *     device error word that mamba_get_device_error() reports.  No call traps
 *     or aborts on the device.
 *   - y must not overlap any input.  u/delta/B/C/A/D may alias one another
 *     (they are only read).
 *   - Not checked (preconditions): A < 0; delta > 0 (delta is the output of
 *     a softplus in the model); finite inputs.
 */
#ifndef MAMBA_SSM_H
#define MAMBA_SSM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st *mamba_stream_t;

typedef enum {
    MAMBA_F32 = 0,  /* float32 */
    MAMBA_BF16 = 1  /* bfloat16 */
} mamba_dtype_t;

typedef enum {
    MAMBA_OK = 0,
    MAMBA_ERR_INVALID_ARG = 1,  /* null required pointer, negative size, unknown dtype, bad alignment */
    MAMBA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (e.g. nstate) */
    MAMBA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    MAMBA_ERR_TIMEOUT = 4       /* a bounded device wait ran out (see mamba_get_device_error) */
} mamba_status_t;

/* Flags for mamba_selective_scan_ex. */
#define MAMBA_SCAN_GENERAL_A 1u  /* never take the path for A[d][n] = (n+1) A[d][0] */
/*
 * Discretisation (default: zero-order hold, section "Ayrık Zamana Geçiş").
 * The Mamba-3 page (bitig.info, "Geliştirilmiş Ayrıklaştırma Şeması") names
 * the Euler method (Mamba-1/2) and the trapezoidal rule (Mamba-3) without
 * formulas; these flags implement the readings
 *   MAMBA_SCAN_EULER      exponential Euler: Abar = exp(Delta A), Bbar = Delta B
 *                         h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t x_t
 *   MAMBA_SCAN_TRAPEZOID  trapezoid rule on the step's input integral:
 *                         h_t = exp(Delta_t A) h_{t-1}
 *                               + Delta_t/2 (exp(Delta_t A) B_{t-1} x_{t-1} + B_t x_t),
 *                         no previous-token term at t = 0 (also with an
 *                         initial state)
 * y_t = C_t . h_t + D x_t in all cases.  Both run the general-A kernel path
 * (one exponential per state); setting both is MAMBA_ERR_INVALID_ARG.
 * mamba_state_update is zero-order hold only.
 */
#define MAMBA_SCAN_EULER 2u
#define MAMBA_SCAN_TRAPEZOID 4u

/*
 * Selective scan over whole sequences (sections "Ayrık Zamana Geçiş" and
 * "Paralel Tarama Algoritması" of the page above), starting from h = 0.
 *
 *   u, delta     device, dtype, [batch][len][channels]       (x_t and Delta_t)
 *   A            device, float32, [channels][nstate]
 *   B, C         device, dtype, [batch][len][nstate]
 *   D            device, float32, [channels], or NULL for no skip term
 *   y            device, dtype, [batch][len][channels]       (output)
 *   final_state  device, float32, [batch][channels][nstate], or NULL; receives
 *                h after the last token (zeros when len == 0)
 *   nstate       number of states per channel: 4, 8, 16 or 32 in this build
 *                (mamba_scan_supported_nstate tells); bf16 with 4 states
 *                loads its tiles without TMA (a B row is 8 bytes)
 *   stream       CUDA stream the work is ordered on
 *
 * Alignment: every pointer must be aligned to its element size; tiles are
 * staged with TMA when u, delta, B and C are 16-byte aligned and a row of
 * channels is a multiple of 16 bytes, with plain loads otherwise.
 * Scratch: every call allocates and frees stream-ordered scratch on `stream`
 * (from a memory pool the library creates on the device, which keeps up to
 * 1 GiB of freed memory for later calls, see mamba_trim_scratch_pool;
 * inside a stream capture, from cudaMallocAsync, and freed with
 * cudaFreeAsync): job counters, the buffer that hands the state from one
 * time chunk to the next, and, when sequences are split into super-chunks
 * that run side by side, their end states and step sums (mamba_scan_plan
 * reports the size).  With super-chunks a third kernel adds the state
 * entering each super-chunk to its outputs; it walks a super-chunk only
 * while that state's decay is at least 2^-32 for MAMBA_F32 data, 2^-20 for
 * MAMBA_BF16 data (the terms left out are below that fraction of their
 * size: under the fp32, resp. bf16, rounding of y; the final state is
 * composed exactly).  batch == 0 or
 * channels == 0 is a no-op that returns MAMBA_OK.
 * The call enqueues only stream-ordered work (allocation, kernels, free), so
 * it can be captured in a CUDA graph once a first call on the device has run
 * outside capture (that call sets the kernels' shared-memory attribute).
 */
int mamba_selective_scan(const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *D,
                         void *y, float *final_state,
                         int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                         int dtype, mamba_stream_t stream);

/*
 * As mamba_selective_scan, plus:
 *   initial_state  device, float32, [batch][channels][nstate], or NULL (zeros):
 *                  the scan resumes from this state (e.g. prefill continued in
 *                  pieces, or a hand-off from recurrent decoding)
 *   chunk_len      > 0: split every sequence into chunks of this many tokens
 *                  (the associative chunk combine is then always used);
 *                  0: chosen automatically
 *   flags          bitwise OR of MAMBA_SCAN_* flags; unknown bits, or EULER
 *                  together with TRAPEZOID, give MAMBA_ERR_INVALID_ARG
 */
int mamba_selective_scan_ex(const void *u, const void *delta, const float *A,
                            const void *B, const void *C, const float *D,
                            const float *initial_state, void *y, float *final_state,
                            int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                            int64_t chunk_len, unsigned flags,
                            int dtype, mamba_stream_t stream);

/*
 * One recurrent step for every (batch, channel) row: the fixed-size-state
 * update used for generation (section "Karmaşıklık Karşılaştırması": the
 * hidden state does not grow with the sequence).  For each row and state n:
 *   h_n <- exp(Delta A_n) h_n + (Delta A_n)^-1 (exp(Delta A_n) - 1) Delta B_n x
 *   y    = sum_n C_n h_n + D x
 *
 *   state   device, float32, [batch][channels][nstate], updated in place
 *   x, delta device, dtype, [batch][channels]
 *   A       device, float32, [channels][nstate]
 *   B, C    device, dtype, [batch][nstate]
 *   D       device, float32, [channels], or NULL
 *   y       device, dtype, [batch][channels] (output; must not overlap inputs)
 *
 * Alignment: state and A 16-byte aligned; B and C aligned to 4 elements;
 * the rest to their element size.  No scratch memory is used.
 */
int mamba_state_update(float *state, const void *x, const void *delta,
                       const float *A, const void *B, const void *C, const float *D,
                       void *y, int64_t batch, int64_t channels, int64_t nstate,
                       int dtype, mamba_stream_t stream);

/*
 * mamba_selective_scan without any device allocation.  (The pages describe
 * no such call; it serves callers of this library, not the method.)
 *
 * Same arguments, layouts, results and asynchrony as mamba_selective_scan.
 * It is for callers that may not allocate device memory inside an operation:
 * inference runtimes and plugin hosts that plan all device memory ahead and
 * hand an operation only its inputs and outputs, deployments held to a fixed
 * memory budget, and processes whose device memory is owned by another
 * allocator (a framework's caching pool), where an allocation made by a
 * library can fail at any point.
 *
 * Its scratch is one file-scope device array of 16 MiB, reserved on every GPU
 * that loads the library until the process exits; it never calls
 * cudaMalloc, cudaMallocAsync or cudaFree.  A problem whose scratch (see
 * mamba_scan_plan: scratch_bytes) exceeds 16 MiB is rejected with
 * MAMBA_ERR_UNSUPPORTED before anything is enqueued; at 16 states that
 * covers, e.g., 8 x 2048 x 3072 and 4 x 8192 x 5120, not 1 x 1,048,576 x 2048.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call uses the same array, which keeps what the previous
 * call left in it: the call clears the parts that must start at zero on
 * `stream`.  Calls that can overlap on the GPU (other streams, other host
 * threads without ordering) race on the array and corrupt each other's
 * results: order them.
 */
int mamba_selective_scan_noalloc(const void *u, const void *delta, const float *A,
                                 const void *B, const void *C, const float *D,
                                 void *y, float *final_state,
                                 int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                                 int dtype, mamba_stream_t stream);

/*
 * mamba_selective_scan on HOST buffers, with the copies overlapped with the
 * scan.  The pages have no counterpart of this call; it serves callers whose
 * sequences live in host memory (prefill from host-resident activations,
 * offline batch scoring).
 *
 *   u, delta, B, C, y, A, D, final_state   host memory, same layouts and
 *                types as mamba_selective_scan (final_state and D may be NULL)
 *   piece_len    > 0: tokens per piece; 0: about len / 8 (at least 256)
 *
 * The sequence is cut into time pieces.  Piece k's host->device copies
 * (cudaMemcpy2DAsync of rows [t0, t0+n) of every batch), its scan and the
 * device->host copy of its y run on one of two streams (`stream` and an
 * internal non-blocking stream, created once per device), so copies overlap
 * the neighbouring pieces' scans; piece k starts from piece k-1's final state
 * (ordered by an event), which is the same recurrence as one scan.
 *
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister): with
 * pageable memory the copies do not overlap.  The call is asynchronous on
 * `stream` (which waits for the internal stream at the end): the host
 * buffers must stay valid, and y / final_state may be read only after
 * `stream` has been synchronised.  Device memory (two pieces' buffers, A, D)
 * is allocated and freed stream-ordered on `stream`.  len == 0 writes zeros
 * to final_state on the host before returning.
 */
int mamba_selective_scan_host(const void *u, const void *delta, const float *A,
                              const void *B, const void *C, const float *D,
                              void *y, float *final_state,
                              int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                              int64_t piece_len, int dtype, mamba_stream_t stream);

/*
 * Backward of the zero-order-hold scan (training): the gradients of
 * L(y, h_final) with respect to every input, given dy = dL/dy and
 * d_final_state = dL/dh_final (NULL: zero).  The pages imply training but
 * print no gradient; this is reverse-mode differentiation of the recurrence
 * of mamba_selective_scan (per state n, z = Delta_t A_n, r = e^z):
 *   lam_t = C_t dy_t + r_{t+1} lam_{t+1}          (the adjoint of h_t)
 *   du_t = sum_n lam_t (r - 1)/A_n B_{t,n} + D dy_t
 *   dDelta_t = sum_n lam_t r (A_n h_{t-1} + B_{t,n} x_t)
 *   dA_n = sum over (b, t) of lam_t (Delta r h_{t-1} + x B Delta^2 psi(z)),
 *          psi(z) = (z e^z - (e^z - 1)) / z^2
 *   dB_{t,n} = sum over channels of lam_t x_t (r - 1)/A_n
 *   dC_{t,n} = sum over channels of dy_t h_t,   dD = sum dy x,   dh0 = r_0 lam_0
 *
 *   u, delta, B, C, dy      device, dtype, layouts as the forward
 *   A, D, initial_state     as the forward (D and initial_state may be NULL)
 *   d_final_state           device, float32, [batch][channels][nstate], or NULL
 *   du, ddelta              device, dtype, [batch][len][channels] (outputs)
 *   dA                      device, float32, [channels][nstate] (output)
 *   dB, dC                  device, float32, [batch][len][nstate] (outputs)
 *   dD                      device, float32, [channels]; required when D is given
 *   d_initial_state         device, float32, [batch][channels][nstate], or NULL
 *   nstate                  4, 8 or 16 (32: MAMBA_ERR_UNSUPPORTED)
 *
 * It runs the forward scan once more, keeping only the state before every
 * tile, then one warp per (batch, 32-channel group) walks the sequence in
 * reverse, recomputing each tile's states from its checkpoint, half a tile at
 * a time (stream-ordered scratch: the checkpoints and [T/2 + 1][32][nstate]
 * floats per warp, T = 64 tokens for bf16 and 32 for float32).  With
 * 16-byte aligned rows (channels * element size and nstate * element size
 * multiples of 16, tensors 16-byte aligned) each tile's inputs are first
 * staged in shared memory (16 KB per warp).  dA, dB,
 * dC and dD are accumulated with atomic adds, so their last bits can vary
 * from call to call.  Asynchronous on `stream`.
 */
int mamba_selective_scan_backward(const void *u, const void *delta, const float *A,
                                  const void *B, const void *C, const float *D,
                                  const float *initial_state, const void *dy,
                                  const float *d_final_state,
                                  void *du, void *ddelta, float *dA, float *dB, float *dC,
                                  float *dD, float *d_initial_state,
                                  int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                                  int dtype, mamba_stream_t stream);

/*
 * Mamba-2's restricted scan in its chunked matrix form (state space duality),
 * on the tensor cores.
 *
 * Defined by: the Mamba-3 page (bitig.info), "Karmaşık Değerli Durum
 * Güncellemesi" (Mamba-2 reduces the state transition to real scalars), and
 * "Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)", "Mamba-2 ve
 * Güncel Gelişmeler" (with that restriction the SSM equals a masked,
 * attention-like matrix form).  Channels are grouped into `heads` heads of
 * `headdim` consecutive channels; head h has one scalar A[h] < 0 and one
 * step dt[b][t][h] shared by its channels, and every channel d of head h
 * runs the selective scan with A[d][n] = A[h] for all n and delta[b][t][d]
 * = dt[b][t][h]:
 *   h_t = exp(dt A) h_{t-1} + w_t B_t x_t,  y_t = C_t . h_t + D x_t,
 *   w_t = (exp(dt A) - 1)/A (zero-order hold) or dt (flag MAMBA_SCAN_EULER).
 * The kernel evaluates it chunk by chunk as matrix products (64-token
 * chunks; the decay-masked C B^T of a chunk times its x, plus the entering
 * state), with bf16 operands and fp32 accumulation; the state carried from
 * chunk to chunk is fp32, its bf16 copy feeds the C . h term.
 *
 * Layouts (row-major, contiguous): x, y [batch][len][heads*headdim] bf16;
 * dt [batch][len][heads] bf16; A [heads] fp32; B, C [batch][len][nstate]
 * bf16 (shared by all heads); D [heads*headdim] fp32 or NULL;
 * initial_state / final_state [batch][heads*headdim][nstate] fp32 or NULL
 * (the selective scan's state layout).  x, B, C and y must be 16-byte
 * aligned, D 8-byte aligned.  All pointers are caller-owned device memory.
 *
 * supers: super-chunks per (batch row, head) run in parallel (0 = chosen
 * from the shape and the device; a forced value is clamped to the chunk
 * count).  With more than one, every super-chunk runs from zero (the first
 * from initial_state) and records its end state (stream-ordered scratch of
 * 4 (64 nstate + 1) bytes per super-chunk and head); a second kernel adds
 * the entering states' effect to y while their decay is at least 2^-20
 * (the terms left out are below 2^-20 of their size, 2^11 times under the
 * bf16 rounding of y) and writes
 * final_state.
 *
 * Supported: dtype MAMBA_BF16, headdim 64, nstate 16, 32 or 64, flags 0 or
 * MAMBA_SCAN_EULER (MAMBA_SCAN_GENERAL_A is accepted and has no effect: A
 * has no state structure here).  Otherwise MAMBA_ERR_UNSUPPORTED
 * (MAMBA_SCAN_TRAPEZOID, fp32 I/O, other headdim or nstate); malformed
 * arguments (NULL tensors with len > 0, negative sizes, misalignment,
 * unknown flags, EULER with TRAPEZOID) give MAMBA_ERR_INVALID_ARG.  len == 0
 * copies initial_state (or zeros) to final_state.  Asynchronous on `stream`.
 */
int mamba_ssd_scan(const void *x, const void *dt, const float *A, const void *B, const void *C,
                   const float *D, const float *initial_state, void *y, float *final_state,
                   int64_t batch, int64_t len, int64_t heads, int64_t headdim, int64_t nstate,
                   int64_t supers, unsigned flags, int dtype, mamba_stream_t stream);

/* 1 if `nstate` is implemented by mamba_ssd_scan. */
int mamba_ssd_supported_nstate(int64_t nstate);

/*
 * The selective scan with a complex diagonal A and a complex state.
 *
 * Defined by: the Mamba-3 page (bitig.info), "Karmaşık Değerli Durum
 * Güncellemesi" (complex state update; complex eigenvalues let the state
 * rotate and oscillate).  The page prints no formula; the reading taken is
 * A[d][n] = A_re[d][n] + i A_im[d][n] (A_re < 0) with the zero-order hold of
 * mamba_selective_scan in complex arithmetic and real B, C:
 *   h_t = exp(delta A) h_{t-1} + (exp(delta A) - 1)/A * B_t x_t
 *   y_t = sum_n C_t[n] Re(h_t[n]) + D x_t
 * so a state turns by delta_t * A_im per token.
 *
 * Layouts as mamba_selective_scan (u, delta, y [batch][len][channels]; B, C
 * [batch][len][nstate]; one dtype for them, fp32 or bf16); A_re, A_im
 * [channels][nstate] fp32; D [channels] fp32 or NULL; initial_state and
 * final_state [batch][channels][nstate][2] fp32 with (re, im) adjacent
 * (8-byte aligned), or NULL.  supers: super-chunks per sequence run in
 * parallel (0 = chosen from the shape and the device); with more than one,
 * stream-ordered scratch of 8 nstate + 8 bytes per (batch, super-chunk,
 * channel) holds their end states and step sums.  nstate 4, 8 or 16
 * (otherwise MAMBA_ERR_UNSUPPORTED).  All arithmetic fp32 (the sum of steps
 * of a super-chunk in double).  Errors and len == 0 as for
 * mamba_selective_scan_ex.  Asynchronous on `stream`.
 */
int mamba_selective_scan_complex(const void *u, const void *delta, const float *A_re,
                                 const float *A_im, const void *B, const void *C, const float *D,
                                 const float *initial_state, void *y, float *final_state,
                                 int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                                 int64_t supers, int dtype, mamba_stream_t stream);

/* 1 if `nstate` is implemented by mamba_selective_scan_complex. */
int mamba_complex_supported_nstate(int64_t nstate);

/*
 * Multi-input multi-output (MIMO) selective scan.
 *
 * Defined by: the Mamba-3 page (bitig.info), "MIMO Mekanizmasının İşleyişi"
 * (the state is updated once per step for several outputs, holds several
 * output predictions without a larger state transition matrix or more
 * parameters) and "Seçici Durum Güncellemesindeki İyileştirmeler" (a
 * separate selective gate per output channel).  The page prints no
 * formula; the reading taken is the zero-order hold of mamba_selective_scan
 * with R inputs and R outputs per channel sharing one state and one step:
 *   h_t = exp(Delta_t A) h_{t-1} + sum_r (Delta_t A)^-1 (exp(Delta_t A) - 1) Delta_t B_t^(r) x_t^(r)
 *   y_t^(r) = C_t^(r) . h_t + D x_t^(r)          (C^(r): the gate of output r)
 *
 *   u, y          device, dtype, [batch][len][ranks][channels]   (x_t^(r), y_t^(r))
 *   delta         device, dtype, [batch][len][channels]          (one step per token and channel)
 *   A             device, float32, [channels][nstate]
 *   B, C          device, dtype, [batch][len][ranks][nstate]     (shared by all channels)
 *   D             device, float32, [channels], or NULL
 *   initial_state, final_state   device, float32, [batch][channels][nstate], or NULL
 *   ranks         R: 2 or 4 in this build, with nstate 16 (mamba_mimo_supported)
 *   flags         0 or MAMBA_SCAN_GENERAL_A (zero-order hold only: EULER or
 *                 TRAPEZOID give MAMBA_ERR_UNSUPPORTED)
 *
 * The same kernels as mamba_selective_scan (a tile of 64/R bf16 or 32/R fp32
 * tokens), the same scratch, asynchrony, alignment and errors;
 * batch * len * ranks must stay below 2^31.
 */
int mamba_selective_scan_mimo(const void *u, const void *delta, const float *A,
                              const void *B, const void *C, const float *D,
                              const float *initial_state, void *y, float *final_state,
                              int64_t batch, int64_t len, int64_t ranks, int64_t channels, int64_t nstate,
                              unsigned flags, int dtype, mamba_stream_t stream);

/*
 * One multi-input multi-output recurrent step for every (batch, channel)
 * row (the decode step of mamba_selective_scan_mimo; the Mamba-3 page says
 * MIMO's point is to serve several outputs per state update):
 *   h_n <- exp(Delta A_n) h_n + (Delta A_n)^-1 (exp(Delta A_n) - 1) Delta sum_r B^(r)_n x^(r)
 *   y^(r) = sum_n C^(r)_n h_n + D x^(r)
 *
 *   state   device, float32, [batch][channels][nstate], updated in place
 *   x, y    device, dtype, [batch][ranks][channels]
 *   delta   device, dtype, [batch][channels]
 *   A       device, float32, [channels][nstate]
 *   B, C    device, dtype, [batch][ranks][nstate]
 *   D       device, float32, [channels], or NULL
 * ranks and nstate as mamba_mimo_supported.  Alignment as mamba_state_update.
 * No scratch memory is used.  Zero-order hold.
 */
int mamba_state_update_mimo(float *state, const void *x, const void *delta,
                            const float *A, const void *B, const void *C, const float *D,
                            void *y, int64_t batch, int64_t ranks, int64_t channels, int64_t nstate,
                            int dtype, mamba_stream_t stream);

/* 1 if mamba_selective_scan_mimo implements this number of inputs/outputs and states. */
int mamba_mimo_supported(int64_t ranks, int64_t nstate);

/* How mamba_selective_scan_ex (zero-order hold, default flags) would split a
 * problem (host-side planning only). */
typedef struct {
    int64_t supers;        /* super-chunks per sequence, run side by side from zero (1: no correction kernel) */
    int64_t super_len;     /* tokens per super-chunk (all but the last) */
    int64_t chunk_len;     /* tokens per job of the chunked kernel */
    int64_t jobs;          /* jobs of the chunked kernel */
    int64_t kernels;       /* kernels one call launches (pre-pass, chunked scan, correction when supers > 1) */
    int64_t scratch_bytes; /* stream-ordered scratch one call allocates */
    int64_t ctas;          /* CTAs of the chunked kernel (persistent: at most one per SM) */
    int64_t consumer_warps; /* consumer warps per CTA: 4, or 8 (two per SM sub-partition) for
                               super-chunks of >= 65,536 tokens of the bf16 zero-order-hold scan
                               with 16 states */
} mamba_scan_plan_t;

/*
 * Fills *out with the split that a scan of this shape would use.
 * sm_count > 0 plans for that many SMs; sm_count <= 0 queries the current
 * device.  Makes no device calls when sm_count > 0.
 */
int mamba_scan_plan(int64_t batch, int64_t len, int64_t channels, int64_t nstate, int64_t chunk_len,
                    int dtype, int sm_count, mamba_scan_plan_t *out);

/* Static description of a status code (never NULL). */
const char *mamba_status_string(int status);

/* 1 if `nstate` is implemented by the scan and state-update kernels. */
int mamba_scan_supported_nstate(int64_t nstate);

/*
 * The device error word of the current device: MAMBA_OK, or MAMBA_ERR_TIMEOUT
 * when a bounded device wait has run out since the word was last cleared.
 * The word is read (and, with clear != 0, reset to MAMBA_OK) by copies
 * enqueued on `stream`, so it reflects every kernel enqueued on `stream`
 * before the call; the call then waits for `stream` alone (it synchronises
 * no other stream, unless `stream` is the legacy default stream, which is
 * ordered with every blocking stream).  MAMBA_ERR_CUDA if a copy or the wait
 * fails.
 */
int mamba_get_device_error(mamba_stream_t stream, int clear);

/*
 * Diagnostic: how many device scratch allocations (stream-ordered, from the
 * library's pool or cudaMallocAsync) the library has made in this process.
 * Lets a test show that a call allocated nothing.
 */
int64_t mamba_debug_scratch_allocations(void);

/*
 * Returns to the system the freed scratch that the library's memory pool on
 * the current device keeps for later calls (up to 1 GiB; see
 * mamba_selective_scan).  Scratch still in use by enqueued work stays.  The
 * pool keeps freed memory because mapping it again on every call costs host
 * time during which the GPU waits; a caller that wants the memory back
 * between phases calls this.  MAMBA_OK, or MAMBA_ERR_CUDA.
 */
int mamba_trim_scratch_pool(void);

/*
 * Diagnostic: enqueues one kernel that waits on a barrier nothing will ever
 * complete, with a wait limit of `limit_ns` nanoseconds (clamped to
 * [1 us, 1 s]).  The wait runs out, the kernel records MAMBA_ERR_TIMEOUT in
 * the device error word and returns normally; the context stays usable.
 * Used by the tests of the timeout path.
 */
int mamba_debug_expire_wait(int64_t limit_ns, mamba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_SSM_H */
