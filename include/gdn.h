/*
 * gdn.h -- C ABI of libgdn, a B200 (sm_100a) implementation of the Gated
 * DeltaNet mixer recurrence.
 *
 * Method (Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t,          alpha_t = exp(g_t)
 *
 * The caller passes the log-decay g (g <= 0); the library applies the
 * exponential itself (same section: the kernel is handed g directly).  The
 * gate is either one value per (token, head) -- GDN_GATE_SCALAR -- or one
 * value per key channel -- GDN_GATE_CHANNEL, the GDN-2 / KDA form ("Gated
 * DeltaNet" entity trail, finding of 2026-07-29).  No 1/sqrt(dk) query scale
 * is applied.  The library neither clamps g nor normalises q and k; both are
 * the caller's contract.
 *
 * Two execution modes compute the same mathematics (entity trail, finding of
 * 2026-07-29: a fused recurrent mode for decode and a chunkwise mode for
 * training / prefill):
 *   gdn_chunk_fwd       chunkwise-parallel prefill over T tokens;
 *   gdn_recurrent_step  one token per sequence, state updated in place.
 *
 * Memory and ownership
 *   Every pointer is caller-owned DEVICE memory (e.g. a torch tensor's
 *   data_ptr()), contiguous and row-major.  q, k, v, out, the states and a
 *   per-channel g must be 16-byte aligned; a scalar g and beta 4-byte
 *   aligned (else GDN_ERR_MISALIGNED).  The library never
 *   frees caller memory.  Scratch space the prefill needs is taken
 *   stream-ordered on `stream` (cudaMallocFromPoolAsync / cudaFreeAsync)
 *   from a memory pool the library creates per device, which keeps its
 *   memory for reuse by later calls (at most the largest scratch in use at
 *   once) until the process ends.
 *   The recurrent state is fp32, [B, H, dk, dv], row index = key channel --
 *   the precision the source keeps the state in ("Hybrid layouts: three
 *   DeltaNet, one attention", section 01 Concept: fp32 recurrent state).
 *
 * Streams and synchronisation
 *   Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream).  No call synchronises the host or the device.
 *
 * Errors
 *   Every argument is validated on the host before anything is launched; an
 *   invalid call returns a negative status and launches nothing.  A launch
 *   failure returns GDN_ERR_CUDA.  A kernel that gives up on a bounded
 *   internal wait records it in a device status word; gdn_check reports it.
 */
#ifndef GDN_H
#define GDN_H

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                        /* = cudaStream_t */
typedef struct CUstream_st* gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1,   /* null required pointer, bad size or enum    */
    GDN_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. dk = 96)   */
    GDN_ERR_MISALIGNED = -3,    /* a pointer is not 16-byte aligned           */
    GDN_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed       */
    GDN_ERR_NOMEM = -5,         /* stream-ordered scratch allocation failed   */
    GDN_ERR_TIMEOUT = -6,       /* a kernel abandoned a bounded wait          */
    GDN_ERR_SCRATCH_LIMIT = -7  /* needs more than the fixed scratch array    */
} gdn_status;

enum { GDN_GATE_SCALAR = 0, GDN_GATE_CHANNEL = 1 };
enum { GDN_IO_BF16 = 0, GDN_IO_F32 = 1 };

/*
 * gdn_chunk_fwd -- chunkwise prefill of T tokens for B sequences and H heads.
 *
 *   q, k      [B, T, H, dk]  bf16 (GDN_IO_BF16, the default)
 *   v         [B, T, H, dv]  bf16
 *   g         [B, T, H] (GDN_GATE_SCALAR) or [B, T, H, dk] (GDN_GATE_CHANNEL),
 *             fp32, g <= 0.  The per-channel gate requires g >= -5, the
 *             domain of the model card's gate parameterisation (section 2.1,
 *             g = -min(softplus(.), 160/bs2) with bs2 = 32); the chunk
 *             factorisation relies on that bound.  The scalar gate accepts
 *             any g <= 0.
 *   beta      [B, T, H] fp32
 *   state_in  [B, H, dk, dv] fp32, or NULL for a zero initial state
 *   out       [B, T, H, dv] fp32; must not alias an input.  fp32 because the
 *             output is a small difference of larger terms: on the source's
 *             workloads max|o| is ~9 rms(o), so bf16 rounding of o alone
 *             would take ~90% of a 2e-2 * rms(o) error budget.
 *   state_out [B, H, dk, dv] fp32, or NULL (final state not written);
 *             state_out == state_in is allowed
 *   dk, dv    64 or 128 (else GDN_ERR_UNSUPPORTED); B, H >= 1; T >= 0.
 *   gate_mode GDN_GATE_SCALAR or GDN_GATE_CHANNEL.
 *   T == 0 writes state_out := state_in (or zeros) and returns GDN_OK; the
 *   per-token pointers (q, k, v, g, beta, out) may then be NULL.
 * Path (bf16, dk = dv = 128): the segment-parallel path of
 * gdn_chunk_fwd_segments where its automatic choice gives n > 1 segments
 * (n = SMs / (B * H) from T > 1984, i.e. 32 chunks, when n >= 3, or with a
 * scalar gate n = 2 with 2 * B * H >= 85% of the SMs), else the prep pool when
 * 2 * B * H <= the SM count, else one CTA per (batch, head).
 * Scratch: the segment path's, as gdn_chunk_fwd_segments (if it cannot be
 * had, the call runs unsegmented).  In the prep pool each chunk's
 * chunk-local results (T' or T and beta, P and the chain's operand tiles:
 * 99,072 bytes) pass from prep CTAs to the state chains through a ring of
 * such records per (batch, head): one per chunk while all of them fit in
 * 256 MiB, else as many as fit (at least 8), whatever T -- at most
 * max(256 MiB, B * H * 8 * 99,072 bytes) plus 4 bytes per record and per
 * (batch, head) of stream-ordered scratch on `stream` from the library's
 * pool, freed on `stream` when the call's kernel completes.  If it cannot be
 * had, the call runs the cluster form of the same kernel, which needs none.
 * After a call that gdn_check reports as GDN_ERR_TIMEOUT, out and state_out
 * are undefined.
 */
GDN_API int gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, const float* state_in, void* out, float* state_out,
                  int B, int T, int H, int dk, int dv, int gate_mode, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_ex -- gdn_chunk_fwd with an explicit I/O dtype and chunk size.
 *   io_dtype   GDN_IO_BF16: q, k, v bf16 (tensor-core chunk path).
 *              GDN_IO_F32 : q, k, v fp32 (fp32 CUDA-core path, for
 *                           tolerances tighter than bf16 operands allow).
 *              out is fp32 in both cases.
 *   chunk_size 0 = default.  bf16: 0 or 64 = chunkwise tensor-core path
 *              (dk = dv = 128; other dims fall back to the token-serial
 *              path when chunk_size is 0), 1 = token-serial fused
 *              recurrence.  fp32: 0 or 1 (token-serial).
 */
GDN_API int gdn_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* state_in, void* out, float* state_out,
                     int B, int T, int H, int dk, int dv, int gate_mode, int io_dtype,
                     int chunk_size, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_segments -- gdn_chunk_fwd (bf16 q, k, v) with explicit
 * sequence parallelism.  The state map of a stretch of tokens is affine,
 * S_end = M S_start + S_end(0) (it follows from the formula of section 2.1),
 * so a long sequence can be cut into num_segments time segments that run in
 * parallel: every segment computes its outputs and end state from a zero
 * start, and its dk x dk transition M with w_t = M_t^T q_t per token; a serial
 * combine gives each segment its true start state, and a correction adds
 * S_start^T w_t to every output.  This costs two chunk passes instead of one
 * and pays off when B * H is small against the SM count and T is long.
 * (gdn_chunk_fwd_segments_noalloc runs the segments a third time from their
 * true starts instead, since w does not fit its fixed scratch.)
 *   num_segments 0 = automatic (what gdn_chunk_fwd does), 1 = none,
 *                n > 1 = n segments (at most one per 64-token chunk;
 *                dk = dv = 128 only).  Automatic: n = SMs / (B * H) from
 *                32 chunks on, when n >= 3, or with a scalar gate n = 2
 *                with 2 * B * H >= 85% of the SMs.  A segment's transition ends once every entry
 *                has decayed below 2^-60 while every token it covers is in
 *                the contracting domain (g <= 0, 0 <= beta <= 1, unit k);
 *                with decaying gates that is after a chunk or two.
 * Scratch: 2 * B * n * H * dk * dv * 4 + B * T * H * dk * 2 bytes (plus
 * 4 bytes per segment), stream-ordered on `stream` from the library's pool
 * (GDN_ERR_NOMEM if it cannot be had with n given; an automatic choice runs
 * unsegmented instead).  Other arguments as gdn_chunk_fwd.
 */
GDN_API int gdn_chunk_fwd_segments(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* state_in, void* out,
                                   float* state_out, int B, int T, int H, int dk, int dv,
                                   int gate_mode, int num_segments, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_segments_noalloc -- gdn_chunk_fwd_segments for callers that
 * must not have the library allocate device memory.  The source pages have
 * no counterpart to this entry point: it is a convenience of this library's
 * interface, computing exactly what gdn_chunk_fwd_segments computes.
 *
 * Who needs it: callers whose device memory already belongs to another
 * allocator (e.g. a framework pool that has reserved all free memory, so a
 * stream-ordered allocation inside the library could fail or fragment it), and callers
 * whose step must never stall in an allocator or fail for lack of memory
 * half-way through.  This variant calls no allocation or free routine: its
 * scratch is a fixed 32 MiB array compiled into the library, which every GPU
 * that loads libgdn holds until the process exits.
 *
 * Limit: the segmented path needs 2 * B * n * H * dk * dv * 4 bytes for n
 * time segments (n = num_segments; automatic, n = SMs / (B * H) when
 * B * H * 4 <= SMs and T > 4032, else 1);
 * with dk = dv = 128 that is B * n * H <= 256.  A larger call returns
 * GDN_ERR_SCRATCH_LIMIT and launches nothing.  With n = 1 no scratch is used.
 * bf16 q, k, v and dk = dv = 128 only (else GDN_ERR_UNSUPPORTED).
 *
 * First call: the first call on a device, with that device current, looks up
 * the device address of the array (once per device); make that first call
 * before any stream capture.
 *
 * Sharing: all calls use the same array and leave their data in it.  A call
 * that completes writes every scratch element before it reads it, so nothing
 * is cleared between calls; after a call that gdn_check reports as
 * GDN_ERR_TIMEOUT (a bounded wait gave up), out and state_out are undefined,
 * since later kernels of that call may read scratch the abandoned pass never
 * wrote.  Two calls whose kernels may run at the same time on
 * one GPU (different streams without ordering between them) race on the
 * array and give wrong results.  Order such calls on one stream.
 * Other arguments as gdn_chunk_fwd_segments.
 */
GDN_API int gdn_chunk_fwd_segments_noalloc(const void* q, const void* k, const void* v,
                                           const float* g, const float* beta,
                                           const float* state_in, void* out, float* state_out,
                                           int B, int T, int H, int dk, int dv, int gate_mode,
                                           int num_segments, gdn_stream_t stream);

/*
 * gdn_recurrent_step -- one decode step for B sequences and H heads.
 *
 *   q, k      [B, H, dk] bf16;   v [B, H, dv] bf16
 *   g         [B, H] or [B, H, dk] fp32 (g <= 0);   beta [B, H] fp32
 *   state_in  [B, H, dk, dv] fp32 (required)
 *   state_out [B, H, dk, dv] fp32 (required); == state_in updates in place
 *   out       [B, H, dv] fp32 (fp32 so that the output keeps the state's
 *             precision); must not alias an input
 */
GDN_API int gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* state_in, float* state_out, void* out,
                       int B, int H, int dk, int dv, int gate_mode, gdn_stream_t stream);

/* gdn_recurrent_step_ex -- io_dtype selects bf16 or fp32 q, k, v; out is fp32. */
GDN_API int gdn_recurrent_step_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* state_in, float* state_out,
                          void* out, int B, int H, int dk, int dv, int gate_mode,
                          int io_dtype, gdn_stream_t stream);

/*
 * gdn_chunk_bwd -- gradients of the chunkwise prefill (training).
 *
 * For the loss sum(d_out * out) + sum(d_state_out * state_out) of the call
 * gdn_chunk_fwd(q, k, v, g, beta, state_in) -> (out, state_out), writes the
 * gradients of every input.  The forward is recomputed inside (chunks of 32
 * tokens: the start state of every chunk, then the state gradient backward
 * over the chunks, then each chunk's token gradients in parallel), in fp32.
 * Reverse mode of the model card's recurrence (section 2.1) in its chunkwise
 * form; the gate enters through a = exp(g) as in the forward.
 *
 *   q, k, v, g, beta, state_in  as gdn_chunk_fwd (bf16 q, k, v; per-channel
 *               g in [-5, 0]; state_in may be NULL = zero)
 *   d_out       [B, T, H, dv] fp32
 *   d_state_out [B, H, dk, dv] fp32, or NULL (zero)
 *   dq, dk      [B, T, H, dk] fp32;  dv [B, T, H, dv] fp32
 *   dg          g's shape, fp32;  dbeta [B, T, H] fp32
 *   d_state_in  [B, H, dk, dv] fp32, or NULL (not written)
 *   No output may overlap an input or another output.  Scratch: about
 *   (T / 32) * B * H * (2 dk dv + 3 * 32 dk + 32 dv + 32^2 + dk) * 4 bytes,
 *   stream-ordered from the library's pool.
 */
GDN_API int gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* state_in, const float* d_out,
                          const float* d_state_out, float* dq, float* dk, float* dv, float* dg,
                          float* dbeta, float* d_state_in, int B, int T, int H, int Dk, int Dv,
                          int gate_mode, gdn_stream_t stream);

/*
 * gdn_recurrent_steps -- T successive tokens per sequence through the decode
 * kernel (speculative verification of T draft tokens; the fused recurrent
 * mode of the "Gated DeltaNet" entity trail, finding of 2026-07-29), with the
 * state after every token optionally kept.
 *
 *   q, k      [B, T, H, dk] bf16;  v [B, T, H, dv] bf16 (token-major, as the
 *             prefill)
 *   g         [B, T, H] or [B, T, H, dk] fp32 (g <= 0);  beta [B, T, H] fp32
 *   state_in  [B, H, dk, dv] fp32 (required)
 *   state_out [B, H, dk, dv] fp32: the state after all T tokens, or NULL;
 *             == state_in updates in place
 *   snapshots [B, T, H, dk, dv] fp32: snapshots[b, t, h] = S_t, the state of
 *             (b, h) after token t, or NULL.  At least one of state_out and
 *             snapshots is required.
 *   out       [B, T, H, dv] fp32
 *   T >= 1; dk, dv 64 or 128.  Results equal T calls of gdn_recurrent_step
 *   (same arithmetic, same order).
 */
GDN_API int gdn_recurrent_steps(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* state_in, float* state_out,
                                float* snapshots, void* out, int B, int T, int H, int dk, int dv,
                                int gate_mode, gdn_stream_t stream);

/*
 * gdn_recurrent_steps_decoupled -- gdn_recurrent_steps with separate erase
 * and write gates: S_t = (I - be_t k_t k_t^T) Diag(a_t) S_{t-1}
 * + bw_t k_t v_t^T.  This is a reading of Gated DeltaNet-2's decoupled
 * erase / write ("Gated DeltaNet" entity trail, finding of 2026-05-22),
 * which gives no formula; be = bw is gdn_recurrent_steps.
 *
 *   beta_erase [B, T, H] fp32 (the erase gate; the beta of the other calls)
 *   beta_write [B, T, H] fp32 (required; must not overlap an output)
 *   every other argument as gdn_recurrent_steps (any T >= 1: one decode step,
 *   draft tokens, or a token-serial prefill).
 */
GDN_API int gdn_recurrent_steps_decoupled(const void* q, const void* k, const void* v,
                                          const float* g, const float* beta_erase,
                                          const float* beta_write, const float* state_in,
                                          float* state_out, float* snapshots, void* out, int B,
                                          int T, int H, int dk, int dv, int gate_mode,
                                          gdn_stream_t stream);

/*
 * gdn_state_select -- commit the accepted prefix of a verification step:
 * state[b] := snapshots[b, n_b - 1] for every sequence b whose accepted
 * count n_b = num_accepted[b] (int32, device memory) lies in 1 .. T; rows
 * with any other count are left as they are.  snapshots as written by
 * gdn_recurrent_steps; state [B, H, dk, dv] fp32 must not overlap them.
 */
GDN_API int gdn_state_select(const float* snapshots, const int* num_accepted, float* state,
                             int B, int T, int H, int dk, int dv, gdn_stream_t stream);

/*
 * The layer's input prologue: what turns the projected inputs of a Gated
 * DeltaNet layer into the recurrence's q, k, v, g and beta.
 *   - A causal depthwise convolution of width 4 over the token axis on every
 *     channel of q | k | v (the DeltaNet layers' kernel-4 convolution, Qwen3.5
 *     27B page, section on the hybrid layout; causal q/k/v convolutions,
 *     HANDOFF timeline page, v2 entry):
 *         y_t[c] = sum_{j=0..3} conv_w[h, c, j] * x_{t-3+j}[c],
 *     tap 3 on the current token.  The inputs before a sequence's first
 *     token come from a 4-slot history ring (slot p mod 4 holds the raw input
 *     of position p) or are zero.
 *   - An activation after the convolution: GDN_ACT_SILU, y / (1 + exp(-y)),
 *     or GDN_ACT_NONE.  The pages name none; SiLU is the usual one.
 *   - q and k L2-normalised per head: x * (sum x^2 + 1e-6)^(-1/2).
 *   - beta = sigmoid(beta_raw); g = -min(softplus(g_raw), 5) (Atomic-GDN2
 *     model card, section 2.1: the bound 160 / bs2 with bs2 = 32).
 * Everything is computed in fp32 from the bf16 / fp32 inputs.
 */
enum { GDN_ACT_NONE = 0, GDN_ACT_SILU = 1 };

/*
 * gdn_prologue -- the prologue over T tokens (prefill), one fused pass.
 *
 *   q_raw, k_raw [B, T, H, dk] bf16;  v_raw [B, T, H, dv] bf16
 *   g_raw      [B, T, H] (GDN_GATE_SCALAR) or [B, T, H, dk] (GDN_GATE_CHANNEL) fp32
 *   beta_raw   [B, T, H] fp32
 *   conv_w     [H, 2 dk + dv, 4] fp32, channels in the order q | k | v
 *   ring       [B, H, 4, 2 dk + dv] fp32 (read for the three positions
 *              before token 0, then slots (pos0 + t) mod 4 of the last
 *              min(T, 4) tokens are overwritten with their raw inputs), or
 *              NULL: zero history, nothing written
 *   pos0       [B] int32 device memory: the position of each row's token 0,
 *              or NULL for all 0.  A position p < 0 reads as zero history.
 *   q, k       [B, T, H, dk] bf16 out;  v [B, T, H, dv] bf16 out
 *   g          same shape as g_raw, fp32 out;  beta [B, T, H] fp32 out
 *   dk, dv     64 or 128; B, H >= 1; T >= 0 (T == 0 does nothing)
 *   activation GDN_ACT_NONE or GDN_ACT_SILU
 * The outputs are what gdn_chunk_fwd takes.  No output may overlap an input,
 * another output or the ring (inputs of a tile are read by its neighbour).
 * conv_w, the q/k/v tensors, the ring and a per-channel g must be 16-byte
 * aligned; a scalar g, beta and pos0 4-byte aligned.
 */
GDN_API int gdn_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                         const float* g_raw, const float* beta_raw, const float* conv_w,
                         float* ring, const int* pos0, void* q, void* k, void* v, float* g,
                         float* beta, int B, int T, int H, int dk, int dv, int gate_mode,
                         int activation, gdn_stream_t stream);

/*
 * gdn_recurrent_step_prologue -- one decode step with the prologue fused
 * into it: the raw inputs of one token per sequence go through the
 * convolution (history from the ring), the activation, the L2 norms and the
 * gate maps inside the decode kernel, which then applies gdn_recurrent_step.
 *
 *   q_raw, k_raw [B, H, dk] bf16;  v_raw [B, H, dv] bf16
 *   g_raw      [B, H] or [B, H, dk] fp32;  beta_raw [B, H] fp32
 *   conv_w     [H, 2 dk + dv, 4] fp32
 *   ring       [B, H, 4, 2 dk + dv] fp32, required: slots pos - 3 .. pos - 1
 *              are read, slot pos mod 4 takes this token's raw input
 *   pos        [B] int32 device memory (the token's position), or NULL for 0
 *   state_in, state_out, out as gdn_recurrent_step (state_out == state_in
 *              updates in place)
 *   dk 64 or 128; dv 64 or 128.
 */
GDN_API int gdn_recurrent_step_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                                        const float* g_raw, const float* beta_raw,
                                        const float* conv_w, float* ring, const int* pos,
                                        const float* state_in, float* state_out, void* out,
                                        int B, int H, int dk, int dv, int gate_mode,
                                        int activation, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_prologue -- the chunkwise prefill of a GDN layer from its raw
 * projections: the prologue above applied while the prefill loads its
 * inputs, then the recurrence (Atomic-GDN2 model card, section 2.1), as
 * gdn_prologue followed by gdn_chunk_fwd on its outputs -- without writing
 * q, k, v, g and beta to memory and reading them back.
 *
 *   q_raw .. pos0, activation   as gdn_prologue (the ring is read for the
 *                               history of token 0 and then updated)
 *   state_in   [B, H, dk, dv] fp32, or NULL for a zero initial state
 *   out        [B, T, H, dv] fp32;  state_out [B, H, dk, dv] fp32 or NULL
 *              (state_out == state_in allowed; out and state_out overlap no
 *              input and not the ring)
 *   fused      0: gdn_prologue into stream-ordered scratch
 *              (B * T * H * (2 dk + dv) * 2 bytes + the gates), then
 *              gdn_chunk_fwd.  1: with dk = dv = 128 and 2 * B * H <= the SM
 *              count, the prologue runs inside the prefill's prep-pool
 *              kernel: the prep tasks convert each chunk's q, k (with the
 *              three earlier tokens of the convolution) and the gates, the
 *              state chains convert v, and only the raw projections are
 *              read; scratch as gdn_chunk_fwd's.  Other shapes (or too few
 *              free SMs) take route 0.  Route 0 is the faster one on B200 at
 *              the GDN-2 layer shape (B 8, T 2048, H 8): the conversion in
 *              the prep tasks costs more than the memory pass it saves.
 * Outputs agree with the two-call sequence to the rounding of the sums of
 * squares; errors and scratch failure as gdn_chunk_fwd.
 */
GDN_API int gdn_chunk_fwd_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                                   const float* g_raw, const float* beta_raw, const float* conv_w,
                                   float* ring, const int* pos0, const float* state_in, void* out,
                                   float* state_out, int B, int T, int H, int dk, int dv,
                                   int gate_mode, int activation, int fused,
                                   gdn_stream_t stream);

/*
 * gdn_check -- synchronises `stream`, then reports GDN_ERR_TIMEOUT if any
 * kernel of this library on the current device abandoned a bounded wait
 * since the last gdn_check (and clears the record), GDN_ERR_CUDA on a CUDA
 * error, else GDN_OK.  This is the only call that synchronises.
 */
GDN_API int gdn_check(gdn_stream_t stream);

/* Human-readable name of a status code (static storage). */
GDN_API const char* gdn_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* GDN_H */
