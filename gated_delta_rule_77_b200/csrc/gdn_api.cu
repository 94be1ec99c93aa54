// gdn_api.cu -- the C ABI of libgdn (declared in include/gdn.h): argument
// validation, dispatch to the kernels, status strings.
//
// Every check runs on the host before anything is launched, so an invalid
// call has no side effect.  Calls never synchronise (except gdn_check).

#include <stdint.h>

#include "../../include/gdn.h"
#include "gdn_internal.cuh"

namespace {

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, size_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}

bool overlaps(Range a, Range b) {
    return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dim_ok(int d) { return d == 64 || d == 128; }

int to_status(cudaError_t e) {
    if (e == cudaSuccess) return GDN_OK;
    return e == cudaErrorMemoryAllocation ? GDN_ERR_NOMEM : GDN_ERR_CUDA;
}

// Shared validation of the tensors of one call.  `T_tokens` is T for the
// prefill and 1 for a decode step (its layout is the T = 1 case).
int validate(const void* q, const void* k, const void* v, const float* g, const float* beta,
             const float* state_in, const float* state_out, const void* out,
             long B, long T_tokens, long H, int dk, int dv, int gate_mode, int io_dtype,
             bool out_f32, bool state_in_required)
{
    // With no tokens the per-token tensors are never touched and may be null.
    if (T_tokens != 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
    if (state_in_required && (!state_in || !state_out)) return GDN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T_tokens < 0 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
    if (gate_mode != GDN_GATE_SCALAR && gate_mode != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (io_dtype != GDN_IO_BF16 && io_dtype != GDN_IO_F32) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    // Keep every element index well inside 64-bit arithmetic and the TMA
    // coordinate range.
    if (B > (1L << 20) || H > (1L << 16) || T_tokens > (1L << 30)) return GDN_ERR_UNSUPPORTED;
    // Rows read or written with vector loads / TMA need 16-byte alignment; a
    // scalar gate and beta are read one float at a time.
    const void* ptrs16[] = {q, k, v, state_in, state_out, out,
                            gate_mode == GDN_GATE_CHANNEL ? g : nullptr};
    for (const void* p : ptrs16)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    for (const void* p : {(const void*)g, (const void*)beta})
        if (p && (reinterpret_cast<uintptr_t>(p) & 3u)) return GDN_ERR_MISALIGNED;

    const size_t esz = io_dtype == GDN_IO_F32 ? 4 : 2;
    const size_t tok = (size_t)B * (size_t)T_tokens * (size_t)H;
    const size_t st = (size_t)B * (size_t)H * (size_t)dk * (size_t)dv * 4;
    const Range rq = range_of(q, tok * dk * esz), rk = range_of(k, tok * dk * esz),
                rv = range_of(v, tok * dv * esz),
                rg = range_of(g, tok * (gate_mode == GDN_GATE_CHANNEL ? dk : 1) * 4),
                rb = range_of(beta, tok * 4),
                ro = range_of(out, tok * dv * (out_f32 ? 4 : esz));
    const Range rsi = state_in ? range_of(state_in, st) : Range{0, 0};
    const Range rso = state_out ? range_of(state_out, st) : Range{0, 0};
    // The output aliases nothing; the final state may only coincide exactly
    // with the initial state.
    for (Range r : {rq, rk, rv, rg, rb, rsi, rso})
        if (overlaps(ro, r)) return GDN_ERR_INVALID_ARG;
    for (Range r : {rq, rk, rv, rg, rb})
        if (overlaps(rso, r)) return GDN_ERR_INVALID_ARG;
    if (state_in && state_out && state_in != state_out && overlaps(rsi, rso))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

// Validation shared by the two prologue entries.  Tensors are listed with
// their sizes; inputs and outputs may not overlap (the ring included).
int validate_prologue(const void* q_raw, const void* k_raw, const void* v_raw, const float* g_raw,
                      const float* beta_raw, const float* conv_w, const float* ring,
                      const int* pos, long B, long T, long H, int dk, int dv, int gate_mode,
                      int activation, const void* const* outs, const size_t* out_bytes, int n_out)
{
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
    if (gate_mode != GDN_GATE_SCALAR && gate_mode != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (activation != GDN_ACT_NONE && activation != GDN_ACT_SILU) return GDN_ERR_INVALID_ARG;
    if (!conv_w) return GDN_ERR_INVALID_ARG;
    if (T != 0) {
        if (!q_raw || !k_raw || !v_raw || !g_raw || !beta_raw) return GDN_ERR_INVALID_ARG;
        for (int i = 0; i < n_out; ++i)
            if (!outs[i]) return GDN_ERR_INVALID_ARG;
    }
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    // The prefill grid is (tiles, H, B): both within the 65535 grid limit.
    if (B > 65535 || H > 65535 || T > (1L << 30)) return GDN_ERR_UNSUPPORTED;
    const bool ch = gate_mode == GDN_GATE_CHANNEL;
    const void* p16[] = {q_raw, k_raw, v_raw, conv_w, ring, ch ? g_raw : nullptr};
    for (const void* p : p16)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    for (const void* p : {(const void*)g_raw, (const void*)beta_raw, (const void*)pos})
        if (p && (reinterpret_cast<uintptr_t>(p) & 3u)) return GDN_ERR_MISALIGNED;
    for (int i = 0; i < n_out; ++i)
        if (outs[i] && !aligned16(outs[i])) return GDN_ERR_MISALIGNED;

    const size_t tok = (size_t)B * (size_t)T * (size_t)H;
    const size_t CH = 2 * (size_t)dk + dv;
    Range in[] = {range_of(q_raw, tok * dk * 2), range_of(k_raw, tok * dk * 2),
                  range_of(v_raw, tok * dv * 2), range_of(g_raw, tok * (ch ? dk : 1) * 4),
                  range_of(beta_raw, tok * 4), range_of(conv_w, (size_t)H * CH * 16),
                  range_of(pos, pos ? (size_t)B * 4 : 0),
                  range_of(ring, ring ? (size_t)B * H * 4 * CH * 4 : 0)};
    const int n_in = sizeof(in) / sizeof(in[0]);
    for (int i = 0; i < n_out; ++i) {
        const Range ro = range_of(outs[i], out_bytes[i]);
        for (int j = 0; j < n_in; ++j)
            if (overlaps(ro, in[j])) return GDN_ERR_INVALID_ARG;
        for (int j = 0; j < i; ++j)
            if (overlaps(ro, range_of(outs[j], out_bytes[j]))) return GDN_ERR_INVALID_ARG;
    }
    // The ring is written: it may not overlap the other inputs either.
    for (int j = 0; j < n_in - 1; ++j)
        if (overlaps(in[n_in - 1], in[j])) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

}  // namespace

extern "C" {

int gdn_prologue(const void* q_raw, const void* k_raw, const void* v_raw, const float* g_raw,
                 const float* beta_raw, const float* conv_w, float* ring, const int* pos0, void* q,
                 void* k, void* v, float* g, float* beta, int B, int T, int H, int dk, int dv,
                 int gate_mode, int activation, gdn_stream_t stream_)
{
    const size_t tok = (size_t)(B > 0 ? B : 0) * (size_t)(T > 0 ? T : 0) * (size_t)(H > 0 ? H : 0);
    const bool ch = gate_mode == GDN_GATE_CHANNEL;
    const void* outs[] = {q, k, v, g, beta};
    const size_t bytes[] = {tok * (size_t)dk * 2, tok * (size_t)dk * 2, tok * (size_t)dv * 2,
                            tok * (ch ? (size_t)dk : 1) * 4, tok * 4};
    int rc = validate_prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, pos0, B, T, H,
                               dk, dv, gate_mode, activation, outs, bytes, 5);
    if (rc != GDN_OK) return rc;
    if (T == 0) return GDN_OK;
    gdn::PrologueArgs a{static_cast<const __nv_bfloat16*>(q_raw),
                        static_cast<const __nv_bfloat16*>(k_raw),
                        static_cast<const __nv_bfloat16*>(v_raw),
                        g_raw, beta_raw, conv_w, ring, pos0, activation == GDN_ACT_SILU,
                        static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
                        static_cast<__nv_bfloat16*>(v), g, beta, B, T, H, dk, dv, ch};
    cudaError_t e = gdn::launch_prologue(a, reinterpret_cast<cudaStream_t>(stream_));
    return e == cudaErrorNotSupported ? GDN_ERR_UNSUPPORTED : to_status(e);
}

int gdn_recurrent_step_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                                const float* g_raw, const float* beta_raw, const float* conv_w,
                                float* ring, const int* pos, const float* state_in,
                                float* state_out, void* out, int B, int H, int dk, int dv,
                                int gate_mode, int activation, gdn_stream_t stream_)
{
    if (!ring || !state_in || !state_out) return GDN_ERR_INVALID_ARG;
    const size_t bh = (size_t)(B > 0 ? B : 0) * (size_t)(H > 0 ? H : 0);
    const size_t st = bh * (size_t)(dk > 0 ? dk : 0) * (size_t)(dv > 0 ? dv : 0) * 4;
    // state_out may coincide with state_in exactly (in-place update); it is
    // then checked once.
    const void* outs[] = {out, state_out};
    const size_t bytes[] = {bh * (size_t)(dv > 0 ? dv : 0) * 4, st};
    int rc = validate_prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, pos, B, 1, H,
                               dk, dv, gate_mode, activation, outs, bytes, 2);
    if (rc != GDN_OK) return rc;
    if (!aligned16(state_in)) return GDN_ERR_MISALIGNED;
    const Range rsi = range_of(state_in, st);
    if (overlaps(rsi, range_of(out, bytes[0]))) return GDN_ERR_INVALID_ARG;
    if (state_in != state_out && overlaps(rsi, range_of(state_out, st))) return GDN_ERR_INVALID_ARG;
    if (overlaps(rsi, range_of(ring, bh * 4 * (2 * (size_t)dk + dv) * 4))) return GDN_ERR_INVALID_ARG;
    gdn::StepPrologueArgs a{static_cast<const __nv_bfloat16*>(q_raw),
                            static_cast<const __nv_bfloat16*>(k_raw),
                            static_cast<const __nv_bfloat16*>(v_raw),
                            g_raw, beta_raw, conv_w, ring, pos, activation == GDN_ACT_SILU,
                            state_in, state_out, static_cast<float*>(out), B, H, dk, dv,
                            gate_mode == GDN_GATE_CHANNEL};
    cudaError_t e = gdn::launch_step_prologue(a, reinterpret_cast<cudaStream_t>(stream_));
    return e == cudaErrorNotSupported ? GDN_ERR_UNSUPPORTED : to_status(e);
}

int gdn_chunk_fwd_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                           const float* g_raw, const float* beta_raw, const float* conv_w, float* ring,
                           const int* pos0, const float* state_in, void* out, float* state_out, int B,
                           int T, int H, int dk, int dv, int gate_mode, int activation,
                           int fused, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (fused != 0 && fused != 1) return GDN_ERR_INVALID_ARG;
    const size_t tok = (size_t)(B > 0 ? B : 0) * (size_t)(T > 0 ? T : 0) * (size_t)(H > 0 ? H : 0);
    const size_t st = (size_t)(B > 0 ? B : 0) * (size_t)(H > 0 ? H : 0) * (size_t)(dk > 0 ? dk : 0) *
                      (size_t)(dv > 0 ? dv : 0) * 4;
    // state_out may coincide with state_in exactly (checked below); out and
    // state_out are outputs that may overlap no input (the ring included).
    const void* outs[] = {out, state_out};
    const size_t bytes[] = {tok * (size_t)(dv > 0 ? dv : 0) * 4, state_out ? st : 0};
    int rc = validate_prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, pos0, B, T, H, dk,
                               dv, gate_mode, activation, outs, bytes, 2);
    if (rc != GDN_OK) return rc;
    if (state_in) {
        if (!aligned16(state_in)) return GDN_ERR_MISALIGNED;
        const Range rsi = range_of(state_in, st);
        if (overlaps(rsi, range_of(out, bytes[0]))) return GDN_ERR_INVALID_ARG;
        if (state_out && state_out != state_in && overlaps(rsi, range_of(state_out, st)))
            return GDN_ERR_INVALID_ARG;
        if (ring && overlaps(rsi, range_of(ring, (size_t)B * H * 4 * (2 * (size_t)dk + dv) * 4)))
            return GDN_ERR_INVALID_ARG;
    }
    if (T > (1 << 30)) return GDN_ERR_UNSUPPORTED;
    if (T == 0) {
        if (!state_out || state_in == state_out) return GDN_OK;
        cudaError_t e = state_in
            ? cudaMemcpyAsync(state_out, state_in, st, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(state_out, 0, st, stream);
        return to_status(e);
    }
    const bool ch = gate_mode == GDN_GATE_CHANNEL;
    gdn::PrologueArgs pa{static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
                         static_cast<const __nv_bfloat16*>(v_raw), g_raw, beta_raw, conv_w, ring, pos0,
                         activation == GDN_ACT_SILU, nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H,
                         dk, dv, ch};
    cudaError_t e = cudaErrorNotSupported;
    if (fused) {
        gdn::ProPrefill fp{pa, state_in, state_out, static_cast<float*>(out)};
        e = gdn::launch_chunk_pool_prologue(fp, stream);
        if (e != cudaErrorNotSupported) return to_status(e);
    }
    // Route 0, or a shape that is not the fused kernel's (or too few free
    // SMs): the prologue pass into stream-ordered scratch, then the prefill.
    const size_t qk = tok * dk * 2, vb = tok * dv * 2, gb = tok * (ch ? (size_t)dk : 1) * 4, bb = tok * 4;
    auto up16 = [](size_t n) { return (n + 255) / 256 * 256; };
    uint8_t* ws = nullptr;
    e = gdn::workspace_alloc(reinterpret_cast<void**>(&ws), 2 * up16(qk) + up16(vb) + up16(gb) + up16(bb),
                             stream);
    if (e != cudaSuccess) return to_status(e);
    pa.q = reinterpret_cast<__nv_bfloat16*>(ws);
    pa.k = reinterpret_cast<__nv_bfloat16*>(ws + up16(qk));
    pa.v = reinterpret_cast<__nv_bfloat16*>(ws + 2 * up16(qk));
    pa.g = reinterpret_cast<float*>(ws + 2 * up16(qk) + up16(vb));
    pa.beta = reinterpret_cast<float*>(ws + 2 * up16(qk) + up16(vb) + up16(gb));
    e = gdn::launch_prologue(pa, stream);
    if (e == cudaSuccess) {
        gdn::Problem p{pa.q, pa.k, pa.v, pa.g, pa.beta, state_in, state_out, out, B, T, H, dk, dv, ch,
                       false, true, 0};
        e = gdn::launch_chunk_sm100(p, stream);
        if (e == cudaErrorNotSupported) e = gdn::launch_recurrent(p, stream);
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    return to_status(e != cudaSuccess ? e : ef);
}

static int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* state_in, void* out, float* state_out,
                          int B, int T, int H, int dk, int dv, int gate_mode, int io_dtype,
                          int chunk_size, int segments, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = validate(q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv, gate_mode,
                      io_dtype, true, false);
    if (rc != GDN_OK) return rc;
    if (segments < 0) return GDN_ERR_INVALID_ARG;
    const bool f32 = io_dtype == GDN_IO_F32;
    if (f32) {
        if (chunk_size != 0 && chunk_size != 1) return GDN_ERR_UNSUPPORTED;
        if (segments > 1) return GDN_ERR_UNSUPPORTED;
    } else if (chunk_size != 0 && chunk_size != 1 && chunk_size != 64) {
        return GDN_ERR_UNSUPPORTED;
    }
    if (segments > 1 && (chunk_size == 1 || dk != 128 || dv != 128)) return GDN_ERR_UNSUPPORTED;
    if (T == 0) {
        if (!state_out) return GDN_OK;
        const size_t st = (size_t)B * H * dk * dv * sizeof(float);
        if (state_in == state_out) return GDN_OK;
        cudaError_t e = state_in
            ? cudaMemcpyAsync(state_out, state_in, st, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(state_out, 0, st, stream);
        return to_status(e);
    }
    gdn::Problem p{q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv,
                   gate_mode == GDN_GATE_CHANNEL, f32, true, segments};
    if (!f32 && chunk_size != 1) {
        cudaError_t e = gdn::launch_chunk_sm100(p, stream);
        if (e != cudaErrorNotSupported) return to_status(e);
        if (chunk_size == 64) return GDN_ERR_UNSUPPORTED;
    }
    return to_status(gdn::launch_recurrent(p, stream));
}

int gdn_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* state_in, void* out, float* state_out,
                     int B, int T, int H, int dk, int dv, int gate_mode, int io_dtype,
                     int chunk_size, gdn_stream_t stream)
{
    return chunk_fwd_impl(q, k, v, g, beta, state_in, out, state_out, B, T, H, dk, dv, gate_mode,
                          io_dtype, chunk_size, 0, stream);
}

int gdn_chunk_fwd_segments(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* state_in, void* out, float* state_out,
                           int B, int T, int H, int dk, int dv, int gate_mode, int num_segments,
                           gdn_stream_t stream)
{
    return chunk_fwd_impl(q, k, v, g, beta, state_in, out, state_out, B, T, H, dk, dv, gate_mode,
                          GDN_IO_BF16, 0, num_segments, stream);
}

int gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, const float* state_in, void* out, float* state_out,
                  int B, int T, int H, int dk, int dv, int gate_mode, gdn_stream_t stream)
{
    return gdn_chunk_fwd_ex(q, k, v, g, beta, state_in, out, state_out, B, T, H, dk, dv,
                            gate_mode, GDN_IO_BF16, 0, stream);
}

int gdn_chunk_fwd_segments_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* state_in, void* out,
                                   float* state_out, int B, int T, int H, int dk, int dv,
                                   int gate_mode, int num_segments, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = validate(q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv, gate_mode,
                      GDN_IO_BF16, true, false);
    if (rc != GDN_OK) return rc;
    if (num_segments < 0) return GDN_ERR_INVALID_ARG;
    if (dk != 128 || dv != 128) return GDN_ERR_UNSUPPORTED;
    if (T == 0) {
        if (!state_out || state_in == state_out) return GDN_OK;
        const size_t st = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = state_in
            ? cudaMemcpyAsync(state_out, state_in, st, cudaMemcpyDeviceToDevice, stream)
            : cudaMemsetAsync(state_out, 0, st, stream);
        return to_status(e);
    }
    gdn::Problem p{q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv,
                   gate_mode == GDN_GATE_CHANNEL, false, true, num_segments};
    bool over_limit = false;
    cudaError_t e = gdn::launch_chunk_sm100_noalloc(p, stream, &over_limit);
    if (over_limit) return GDN_ERR_SCRATCH_LIMIT;
    return to_status(e);
}

int gdn_recurrent_step_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* state_in, float* state_out,
                          void* out, int B, int H, int dk, int dv, int gate_mode,
                          int io_dtype, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = validate(q, k, v, g, beta, state_in, state_out, out, B, 1, H, dk, dv, gate_mode,
                      io_dtype, true, true);
    if (rc != GDN_OK) return rc;
    gdn::Problem p{q, k, v, g, beta, state_in, state_out, out, B, 1, H, dk, dv,
                   gate_mode == GDN_GATE_CHANNEL, io_dtype == GDN_IO_F32, true};
    return to_status(gdn::launch_recurrent(p, stream));
}

int gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* state_in, float* state_out, void* out,
                       int B, int H, int dk, int dv, int gate_mode, gdn_stream_t stream)
{
    return gdn_recurrent_step_ex(q, k, v, g, beta, state_in, state_out, out, B, H, dk, dv,
                                 gate_mode, GDN_IO_BF16, stream);
}

static int recurrent_steps_impl(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* beta_write, const float* state_in,
                                float* state_out, float* snapshots, void* out, int B, int T, int H,
                                int dk, int dv, int gate_mode, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!state_in || T < 1) return GDN_ERR_INVALID_ARG;
    if (!state_out && !snapshots) return GDN_ERR_INVALID_ARG;   // nothing would be kept
    int rc = validate(q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv, gate_mode,
                      GDN_IO_BF16, true, false);
    if (rc != GDN_OK) return rc;
    if (snapshots) {
        if (!aligned16(snapshots)) return GDN_ERR_MISALIGNED;
        const size_t tok = (size_t)B * T * H;
        const size_t st = (size_t)B * H * dk * dv * 4;
        const Range rs = range_of(snapshots, tok * dk * dv * 4);
        const bool ch = gate_mode == GDN_GATE_CHANNEL;
        const Range others[] = {range_of(q, tok * dk * 2), range_of(k, tok * dk * 2),
                                range_of(v, tok * dv * 2), range_of(g, tok * (ch ? dk : 1) * 4),
                                range_of(beta, tok * 4), range_of(out, tok * dv * 4),
                                range_of(state_in, st),
                                state_out ? range_of(state_out, st) : Range{0, 0}};
        for (Range r : others)
            if (overlaps(rs, r)) return GDN_ERR_INVALID_ARG;
    }
    gdn::Problem p{q, k, v, g, beta, state_in, state_out, out, B, T, H, dk, dv,
                   gate_mode == GDN_GATE_CHANNEL, false, true};
    p.snapshots = snapshots;
    p.beta_write = beta_write;
    return to_status(gdn::launch_recurrent(p, stream));
}

int gdn_recurrent_steps(const void* q, const void* k, const void* v, const float* g,
                        const float* beta, const float* state_in, float* state_out,
                        float* snapshots, void* out, int B, int T, int H, int dk, int dv,
                        int gate_mode, gdn_stream_t stream_)
{
    return recurrent_steps_impl(q, k, v, g, beta, nullptr, state_in, state_out, snapshots, out, B, T,
                                H, dk, dv, gate_mode, stream_);
}

int gdn_recurrent_steps_decoupled(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta_erase, const float* beta_write,
                                  const float* state_in, float* state_out, float* snapshots,
                                  void* out, int B, int T, int H, int dk, int dv, int gate_mode,
                                  gdn_stream_t stream_)
{
    if (!beta_write) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(beta_write) & 3u) return GDN_ERR_MISALIGNED;
    if (B >= 1 && T >= 1 && H >= 1) {
        const size_t tok = (size_t)B * T * H;
        const Range rw = range_of(beta_write, tok * 4);
        const Range outs[] = {range_of(out, tok * (size_t)(dv > 0 ? dv : 0) * 4),
                              state_out ? range_of(state_out, (size_t)B * H * dk * dv * 4) : Range{0, 0},
                              snapshots ? range_of(snapshots, tok * (size_t)dk * dv * 4) : Range{0, 0}};
        for (Range r : outs)
            if (overlaps(rw, r)) return GDN_ERR_INVALID_ARG;
    }
    return recurrent_steps_impl(q, k, v, g, beta_erase, beta_write, state_in, state_out, snapshots,
                                out, B, T, H, dk, dv, gate_mode, stream_);
}

int gdn_state_select(const float* snapshots, const int* num_accepted, float* state, int B, int T,
                     int H, int dk, int dv, gdn_stream_t stream_)
{
    if (!snapshots || !num_accepted || !state) return GDN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 1) return GDN_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || (long)B * H > 2147483647L) return GDN_ERR_UNSUPPORTED;
    if (!aligned16(snapshots) || !aligned16(state)) return GDN_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(num_accepted) & 3u) return GDN_ERR_MISALIGNED;
    const size_t st = (size_t)B * H * dk * dv * 4;
    const Range rst = range_of(state, st);
    if (overlaps(rst, range_of(snapshots, st * T)) || overlaps(rst, range_of(num_accepted, (size_t)B * 4)))
        return GDN_ERR_INVALID_ARG;
    return to_status(gdn::launch_state_select(snapshots, num_accepted, state, B, T, H, dk, dv,
                                              reinterpret_cast<cudaStream_t>(stream_)));
}

int gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const float* state_in, const float* d_out, const float* d_state_out, float* dq,
                  float* dk, float* dv, float* dg, float* dbeta, float* d_state_in, int B, int T,
                  int H, int Dk, int Dv, int gate_mode, gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (B < 1 || H < 1 || T < 0 || Dk < 1 || Dv < 1) return GDN_ERR_INVALID_ARG;
    if (gate_mode != GDN_GATE_SCALAR && gate_mode != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !d_out || !dq || !dk || !dv || !dg || !dbeta))
        return GDN_ERR_INVALID_ARG;
    if (!dim_ok(Dk) || !dim_ok(Dv)) return GDN_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || T > (1L << 30)) return GDN_ERR_UNSUPPORTED;
    const bool ch = gate_mode == GDN_GATE_CHANNEL;
    const void* p16[] = {q, k, v, d_out, state_in, d_state_out, dq, dk, dv, d_state_in,
                         ch ? (const void*)g : nullptr, ch ? (const void*)dg : nullptr};
    for (const void* ptr : p16)
        if (ptr && !aligned16(ptr)) return GDN_ERR_MISALIGNED;
    for (const void* ptr : {(const void*)g, (const void*)beta, (const void*)dg, (const void*)dbeta})
        if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 3u)) return GDN_ERR_MISALIGNED;
    const size_t tok = (size_t)B * T * H;
    const size_t st = (size_t)B * H * Dk * Dv * 4;
    const size_t gw = ch ? (size_t)Dk : 1;
    const Range in[] = {range_of(q, tok * Dk * 2), range_of(k, tok * Dk * 2), range_of(v, tok * Dv * 2),
                        range_of(g, tok * gw * 4), range_of(beta, tok * 4), range_of(d_out, tok * Dv * 4),
                        state_in ? range_of(state_in, st) : Range{0, 0},
                        d_state_out ? range_of(d_state_out, st) : Range{0, 0}};
    const Range out[] = {range_of(dq, tok * Dk * 4), range_of(dk, tok * Dk * 4), range_of(dv, tok * Dv * 4),
                         range_of(dg, tok * gw * 4), range_of(dbeta, tok * 4),
                         d_state_in ? range_of(d_state_in, st) : Range{0, 0}};
    for (int i = 0; i < 6; ++i) {
        for (Range r : in)
            if (overlaps(out[i], r)) return GDN_ERR_INVALID_ARG;
        for (int j = 0; j < i; ++j)
            if (overlaps(out[i], out[j])) return GDN_ERR_INVALID_ARG;
    }
    if (T == 0) {   // the state passes through unchanged
        if (!d_state_in) return GDN_OK;
        cudaError_t e = d_state_out ? cudaMemcpyAsync(d_state_in, d_state_out, st, cudaMemcpyDeviceToDevice, stream)
                                    : cudaMemsetAsync(d_state_in, 0, st, stream);
        return to_status(e);
    }
    gdn::BwdProblem p{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                      static_cast<const __nv_bfloat16*>(v), g, beta, state_in, d_out, d_state_out,
                      dq, dk, dv, dg, dbeta, d_state_in, B, T, H, Dk, Dv, ch};
    cudaError_t e = gdn::launch_chunk_bwd(p, stream);
    return e == cudaErrorNotSupported ? GDN_ERR_UNSUPPORTED : to_status(e);
}

int gdn_check(gdn_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    unsigned int status = 0;
    cudaError_t e = gdn::read_and_clear_status(&status, stream);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    return status ? GDN_ERR_TIMEOUT : GDN_OK;
}

const char* gdn_status_string(int status)
{
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_MISALIGNED: return "GDN_ERR_MISALIGNED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_NOMEM: return "GDN_ERR_NOMEM";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_SCRATCH_LIMIT: return "GDN_ERR_SCRATCH_LIMIT";
        default: return "GDN_ERR_UNKNOWN";
    }
}

}  // extern "C"
