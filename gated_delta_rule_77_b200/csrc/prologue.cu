// prologue.cu -- the layer's input prologue ahead of the recurrence, fused.
//
// From the projected inputs q_raw, k_raw, v_raw (bf16) and the raw gates:
//   * a causal depthwise convolution of width 4 over the token axis on every
//     channel of q | k | v (the DeltaNet layers' "kernel-4 convolution",
//     Qwen3.5 27B page, hybrid-layout section; causal convolutions on q/k/v,
//     HANDOFF timeline page, v2 entry), tap 3 on the current token, with the
//     three earlier positions taken from a 4-slot history ring (slot p mod 4
//     holds position p's raw input) or zero;
//   * SiLU after the convolution, or none;
//   * q and k L2-normalised per head: x (sum x^2 + 1e-6)^(-1/2);
//   * beta = sigmoid(beta_raw), g = -min(softplus(g_raw), 5) (Atomic-GDN2
//     model card, section 2.1, bound 160 / bs2 with bs2 = 32).
//
// Two forms.  Prefill: one HBM-bound pass (prologue_kernel) writes q, k, v
// (bf16) and g, beta (fp32) for the chunk kernels, then prologue_ring_kernel
// writes the ring (a second launch, so that the ring can be read and written
// by the same call).  Decode: recurrent_prologue_kernel is the fused decode
// step with the prologue in its staging: the step's inputs never leave the
// SM, and the ring write (slot p mod 4) touches no slot that the step reads.

#include <math.h>

#include "chunk_common.cuh"
#include "gdn_internal.cuh"
#include "prologue_math.cuh"

namespace gdn {
namespace {

constexpr int TT = 16;   // tokens per CTA of the prefill prologue (a multiple of 8)

using namespace prologue_math;

// Channels c of q | k | v for token t of row b, head h (bf16 inputs).
__device__ __forceinline__ float2 raw_pair(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                           const __nv_bfloat16* v, long tok, int c, int dk, int dv) {
    const __nv_bfloat16* src;
    long i;
    if (c < dk) { src = q; i = tok * dk + c; }
    else if (c < 2 * dk) { src = k; i = tok * dk + (c - dk); }
    else { src = v; i = tok * dv + (c - 2 * dk); }
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(src + i);
    return __bfloat1622float2(x);
}

// 16 bytes (8 channels) of the raw row q | k | v of one token.
__device__ __forceinline__ uint4 raw16(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                       const __nv_bfloat16* v, long tok, int c, int dk, int dv) {
    const __nv_bfloat16* src;
    long i;
    if (c < dk) { src = q; i = tok * dk + c; }
    else if (c < 2 * dk) { src = k; i = tok * dk + (c - dk); }
    else { src = v; i = tok * dv + (c - 2 * dk); }
    return *reinterpret_cast<const uint4*>(src + i);
}

// One CTA: TT tokens of one (batch, head).
//   1. Stage: every thread issues its 16-byte loads of the raw rows of the
//      tile (and the three rows before it, from the inputs or the ring) and
//      of the gate, before any is used; the rows go to shared memory.
//   2. Convolve: one thread per pair of channels slides the 4-tap window
//      down the tile; the activations stay in registers.  The sums of
//      squares of q and k per token go through warp shuffles and one
//      exchange in shared memory.
//   3. Normalise, write the bf16 results over the staged rows (each thread
//      its own channels), and store the rows back with 16-byte stores.
template <int DK, int DV, bool CHANNEL, int TT>
__global__ void __launch_bounds__((2 * DK + DV) / 2)
prologue_kernel(const __nv_bfloat16* __restrict__ q_raw, const __nv_bfloat16* __restrict__ k_raw,
                const __nv_bfloat16* __restrict__ v_raw, const float* __restrict__ g_raw,
                const float* __restrict__ beta_raw, const float* __restrict__ conv_w,
                const float* __restrict__ ring, const int* __restrict__ pos0, bool silu,
                __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v,
                float* __restrict__ g, float* __restrict__ beta, int T, int H)
{
    constexpr int CH = 2 * DK + DV;
    constexpr int NT = CH / 2;                  // threads
    constexpr int QW = DK / 64;                 // warps per q (and per k)
    constexpr int CPR = CH / 8;                 // 16-byte chunks per token row
    constexpr int NX = TT * CPR;                // chunks of the tile
    constexpr int PX = (NX + NT - 1) / NT;      // chunks per thread
    constexpr int NG = CHANNEL ? TT * DK / 4 : 0;   // float4 of the per-channel gate
    constexpr int PG = CHANNEL ? (NG + NT - 1) / NT : 0;
    static_assert(3 * CPR <= NT && TT <= NT, "staging layout");

    __shared__ __align__(16) __nv_bfloat16 s_x[TT][CH];   // raw rows, then results
    __shared__ __align__(16) float s_h[3][CH];            // the three rows before the tile
    __shared__ float s_ss[2][QW][TT];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * TT, h = blockIdx.y, b = blockIdx.z;
    const int nt = min(TT, T - t0);
    auto tok_of = [&](int t) -> long { return ((long)b * T + t) * H + h; };

    // ---- 1. stage (all loads first) ----
    uint4 xb[PX];
#pragma unroll
    for (int j = 0; j < PX; ++j) {
        const int idx = tid + j * NT;
        const int i = idx / CPR, cc = (idx % CPR) * 8;
        xb[j] = make_uint4(0u, 0u, 0u, 0u);
        if (idx < NX && i < nt) xb[j] = raw16(q_raw, k_raw, v_raw, tok_of(t0 + i), cc, DK, DV);
    }
    float hb[8];
    const int hr = tid / CPR, hc = (tid % CPR) * 8;
    if (tid < 3 * CPR) {
        const int t = t0 - 3 + hr;
        if (t >= 0) {
            const uint4 u = raw16(q_raw, k_raw, v_raw, tok_of(t), hc, DK, DV);
            const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float2 f = __bfloat1622float2(e[m]);
                hb[2 * m] = f.x; hb[2 * m + 1] = f.y;
            }
        } else {
            const int p = (pos0 ? pos0[b] : 0) + t;
#pragma unroll
            for (int m = 0; m < 8; ++m) hb[m] = 0.f;
            if (ring != nullptr && p >= 0) {
                const float* r = ring + (((long)b * H + h) * 4 + (p & 3)) * CH + hc;
                const float4 f0 = *reinterpret_cast<const float4*>(r);
                const float4 f1 = *reinterpret_cast<const float4*>(r + 4);
                hb[0] = f0.x; hb[1] = f0.y; hb[2] = f0.z; hb[3] = f0.w;
                hb[4] = f1.x; hb[5] = f1.y; hb[6] = f1.z; hb[7] = f1.w;
            }
        }
    }
    float4 gb[PG > 0 ? PG : 1];
    if constexpr (CHANNEL) {
#pragma unroll
        for (int j = 0; j < PG; ++j) {
            const int idx = tid + j * NT;
            const int i = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
            gb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (idx < NG && i < nt)
                gb[j] = *reinterpret_cast<const float4*>(g_raw + tok_of(t0 + i) * DK + c4);
        }
    }
    float braw = 0.f, graw = 0.f;
    if (tid < nt) {
        braw = beta_raw[tok_of(t0 + tid)];
        if (!CHANNEL) graw = g_raw[tok_of(t0 + tid)];
    }

#pragma unroll
    for (int j = 0; j < PX; ++j) {
        const int idx = tid + j * NT;
        if (idx < NX) *reinterpret_cast<uint4*>(&s_x[idx / CPR][(idx % CPR) * 8]) = xb[j];
    }
    if (tid < 3 * CPR) {
        *reinterpret_cast<float4*>(&s_h[hr][hc]) = make_float4(hb[0], hb[1], hb[2], hb[3]);
        *reinterpret_cast<float4*>(&s_h[hr][hc + 4]) = make_float4(hb[4], hb[5], hb[6], hb[7]);
    }
    // The gate maps need nothing staged: apply and store them now.
    if constexpr (CHANNEL) {
#pragma unroll
        for (int j = 0; j < PG; ++j) {
            const int idx = tid + j * NT;
            const int i = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
            if (idx < NG && i < nt)
                *reinterpret_cast<float4*>(g + tok_of(t0 + i) * DK + c4) =
                    [&] {
                        const float2 lo = gate_fn2(make_float2(gb[j].x, gb[j].y));
                        const float2 hi = gate_fn2(make_float2(gb[j].z, gb[j].w));
                        return make_float4(lo.x, lo.y, hi.x, hi.y);
                    }();
        }
    }
    if (tid < nt) {
        beta[tok_of(t0 + tid)] = sigmoid_fn(braw);
        if (!CHANNEL) g[tok_of(t0 + tid)] = gate_fn(graw);
    }
    __syncthreads();

    // ---- 2. convolve ----
    const int c = 2 * tid;
    const float4 w0 = *reinterpret_cast<const float4*>(conv_w + ((long)h * CH + c) * 4);
    const float4 w1 = *reinterpret_cast<const float4*>(conv_w + ((long)h * CH + c + 1) * 4);
    float2 win[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) win[r] = make_float2(s_h[r][c], s_h[r][c + 1]);
    // Taps of the two channels side by side, for paired arithmetic.
    const float2 ta = make_float2(w0.x, w1.x), tb = make_float2(w0.y, w1.y);
    const float2 tc = make_float2(w0.z, w1.z), td = make_float2(w0.w, w1.w);
    float2 y[TT];
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&s_x[i][c]));
        const float2 a = fma2(ta, win[0], fma2(tb, win[1], fma2(tc, win[2], mul2(td, x))));
        y[i] = act_fn2(a, silu);
        win[0] = win[1]; win[1] = win[2]; win[2] = x;
    }
    const int tensor = warp / QW;               // 0 q, 1 k, >= 2 v
    if (tensor < 2) {
        // Sums of squares of the TT = 16 tokens over the warp's 32 lanes by a
        // transposing butterfly: at each step a lane keeps half of its
        // remaining tokens and adds its partner's partial for them, so that
        // 8 + 4 + 2 + 1 + 1 shuffles leave lanes 2j and 2j + 1 with the
        // warp's total for one token.
        static_assert(TT == 16, "the butterfly below is written for 16 tokens");
        float v[TT];
#pragma unroll
        for (int i = 0; i < TT; ++i) v[i] = fmaf(y[i].x, y[i].x, y[i].y * y[i].y);
        butterfly_sums16(v, lane);
        if ((lane & 1) == 0) s_ss[tensor][warp % QW][butterfly_token(lane)] = v[0];
    }
    __syncthreads();

    // ---- 3. normalise, write over the staged rows, store ----
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        float2 o = y[i];
        if (tensor < 2) {
            float ss = 0.f;
#pragma unroll
            for (int wq = 0; wq < QW; ++wq) ss += s_ss[tensor][wq][i];
            const float inv = rsqrtf(ss + 1e-6f);
            o.x *= inv; o.y *= inv;
        }
        *reinterpret_cast<__nv_bfloat162*>(&s_x[i][c]) = __floats2bfloat162_rn(o.x, o.y);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < PX; ++j) {
        const int idx = tid + j * NT;
        const int i = idx / CPR, cc = (idx % CPR) * 8;
        if (idx < NX && i < nt) {
            const uint4 u = *reinterpret_cast<const uint4*>(&s_x[i][cc]);
            const long tok = tok_of(t0 + i);
            __nv_bfloat16* dst = cc < DK ? q + tok * DK + cc
                               : cc < 2 * DK ? k + tok * DK + (cc - DK) : v + tok * DV + (cc - 2 * DK);
            *reinterpret_cast<uint4*>(dst) = u;
        }
    }
}

// Ring after the call: slot (p0 + t) mod 4 <- raw input of token t, for the
// last min(T, 4) tokens; other slots unchanged.
template <int DK, int DV>
__global__ void prologue_ring_kernel(const __nv_bfloat16* __restrict__ q_raw,
                                     const __nv_bfloat16* __restrict__ k_raw,
                                     const __nv_bfloat16* __restrict__ v_raw, float* __restrict__ ring,
                                     const int* __restrict__ pos0, int T, int H)
{
    constexpr int CH = 2 * DK + DV;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int p0 = pos0 ? pos0[b] : 0;
    for (int c = 2 * threadIdx.x; c < CH; c += 2 * blockDim.x) {
        for (int t = max(0, T - 4); t < T; ++t) {
            const float2 x = raw_pair(q_raw, k_raw, v_raw, ((long)b * T + t) * H + h, c, DK, DV);
            float* r = ring + (((long)b * H + h) * 4 + ((p0 + t) & 3)) * CH + c;
            r[0] = x.x;
            r[1] = x.y;
        }
    }
}

// Decode step with the prologue fused into its staging (one token per call).
// Tiling as the decode kernel (recurrent.cu): one CTA per (batch, head, slice
// of COLS value columns), the state slice in registers.  Thread i < DK maps
// channel i of q and of k; the L2 norms are one block reduction.  Ring: every
// CTA reads slots p-3 .. p-1; slot p mod 4 is written (q, k channels by slice
// 0, v columns by the slice that owns them), so no CTA writes what another
// reads in the same call.
template <int DK, int COLS, int NWARPS, bool CHANNEL>
__global__ void __launch_bounds__(NWARPS * 32, 5)   // 5 CTAs per SM: measured faster than 4
recurrent_prologue_kernel(const __nv_bfloat16* __restrict__ q_raw, const __nv_bfloat16* __restrict__ k_raw,
                          const __nv_bfloat16* __restrict__ v_raw, const float* __restrict__ g_raw,
                          const float* __restrict__ beta_raw, const float* __restrict__ conv_w,
                          float* ring, const int* __restrict__ pos, bool silu,
                          const float* state_in, float* state_out, float* __restrict__ out, int H, int dv)
{
    constexpr int VW = COLS / 32;
    constexpr int R = DK / NWARPS;
    constexpr int NT = NWARPS * 32;
    static_assert(COLS % 32 == 0 && VW <= 2 && DK % NWARPS == 0 && DK <= NT, "bad tiling");

    __shared__ float s_q[DK];
    __shared__ float s_k[DK];
    __shared__ float s_a[CHANNEL ? DK : 1];
    __shared__ float s_red[2][NWARPS][COLS];
    __shared__ float s_kq[NWARPS];
    __shared__ float s_ss[2][NWARPS];

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int nslices = dv / COLS;
    const int slice = blockIdx.x % nslices;
    const int h = (blockIdx.x / nslices) % H;
    const int b = blockIdx.x / nslices / H;
    const int col0 = slice * COLS + lane * VW;
    const int row0 = warp * R;
    const int CH = 2 * DK + dv;
    const int p = pos ? pos[b] : 0;
    const long tok = (long)b * H + h;
    const long ring_bh = ((long)b * H + h) * 4;

    // The state slice first (8-byte loads, the bulk of the traffic), then the
    // prologue's loads, none of which waits on another: the ring is read in
    // all four slots and the three history slots are picked afterwards.
    float s[R][VW];
    const long sbase = ((long)b * H + h) * DK * (long)dv;
    if (state_in != nullptr) {      // one test outside the loop: every load issued back to back
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if constexpr (VW == 2) {
                const float2 t = *reinterpret_cast<const float2*>(state_in + sbase + (long)(row0 + r) * dv + col0);
                s[r][0] = t.x; s[r][1] = t.y;
            } else {
                s[r][0] = state_in[sbase + (long)(row0 + r) * dv + col0];
            }
        }
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < VW; ++c) s[r][c] = 0.f;
    }

    // Convolution of one channel: taps 0..2 from ring slots p-3 .. p-1 (zero
    // before position 0), tap 3 the input.
    auto conv1 = [&](int ch, float x) -> float {
        const float4 w = *reinterpret_cast<const float4*>(conv_w + ((long)h * CH + ch) * 4);
        float sl[4] = {0.f, 0.f, 0.f, 0.f};
        if (ring) {
#pragma unroll
            for (int j = 0; j < 4; ++j) sl[j] = ring[(ring_bh + j) * CH + ch];
        }
        float hst[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int pp = p - 3 + j;
            const int m = pp & 3;
            const float val = m == 0 ? sl[0] : m == 1 ? sl[1] : m == 2 ? sl[2] : sl[3];
            hst[j] = pp >= 0 ? val : 0.f;
        }
        return act_fn(w.x * hst[0] + w.y * hst[1] + w.z * hst[2] + w.w * x, silu);
    };

    float yq = 0.f, yk = 0.f;
    if (tid < DK) {
        const float xq = __bfloat162float(q_raw[tok * DK + tid]);
        const float xk = __bfloat162float(k_raw[tok * DK + tid]);
        yq = conv1(tid, xq);
        yk = conv1(DK + tid, xk);
        if (CHANNEL) s_a[tid] = expf(gate_fn(g_raw[tok * DK + tid]));
        if (ring && slice == 0) {
            ring[(ring_bh + (p & 3)) * CH + tid] = xq;
            ring[(ring_bh + (p & 3)) * CH + DK + tid] = xk;
        }
    }
    if (tid < DK) {           // unnormalised: the norms are applied after the reductions
        s_q[tid] = yq;
        s_k[tid] = yk;
    }
    float vv[VW];
#pragma unroll
    for (int c = 0; c < VW; ++c) {
        const float xv = __bfloat162float(v_raw[tok * dv + col0 + c]);
        vv[c] = conv1(2 * DK + col0 + c, xv);
        if (ring && warp == 0) ring[(ring_bh + (p & 3)) * CH + 2 * DK + col0 + c] = xv;
    }
    const float bt = sigmoid_fn(beta_raw[tok]);
    float a_scalar = 1.f;
    if (!CHANNEL) a_scalar = expf(gate_fn(g_raw[tok]));
    __syncthreads();

    // The decode step (as recurrent.cu) with q = yq / |yq|, k = yk / |yk|.
    // The norms are scalars of the head, so they are applied after the
    // column reductions: x = S'^T yk / |yk|, c = S'^T yq / |yq|, and their
    // sums of squares ride along in the same exchange.  S' = Diag(a) S,
    // u = b (v - x), S = S' + k u^T, o = c + u (k . q).
    float px[VW], pc[VW];
#pragma unroll
    for (int c = 0; c < VW; ++c) { px[c] = 0.f; pc[c] = 0.f; }
    float kq = 0.f, ssk = 0.f, ssq = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float ki = s_k[row0 + r];
        const float qi = s_q[row0 + r];
        const float ai = CHANNEL ? s_a[row0 + r] : a_scalar;
        kq = fmaf(ki, qi, kq);
        ssk = fmaf(ki, ki, ssk);
        ssq = fmaf(qi, qi, ssq);
#pragma unroll
        for (int c = 0; c < VW; ++c) {
            s[r][c] *= ai;
            px[c] = fmaf(ki, s[r][c], px[c]);
            pc[c] = fmaf(qi, s[r][c], pc[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < VW; ++c) {
        s_red[0][warp][lane * VW + c] = px[c];
        s_red[1][warp][lane * VW + c] = pc[c];
    }
    if (lane == 0) {
        s_kq[warp] = kq;
        s_ss[0][warp] = ssq;
        s_ss[1][warp] = ssk;
    }
    __syncthreads();
    float kq_all = 0.f, nq = 0.f, nk = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
        kq_all += s_kq[w];
        nq += s_ss[0][w];
        nk += s_ss[1][w];
    }
    const float iq = rsqrtf(nq + 1e-6f), ik = rsqrtf(nk + 1e-6f);
    float u[VW];
#pragma unroll
    for (int c = 0; c < VW; ++c) {
        float x = 0.f, cc = 0.f;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) {
            x += s_red[0][w][lane * VW + c];
            cc += s_red[1][w][lane * VW + c];
        }
        u[c] = bt * (vv[c] - x * ik);
        if (warp == 0) out[tok * dv + col0 + c] = fmaf(u[c], kq_all * ik * iq, cc * iq);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float ki = s_k[row0 + r] * ik;
#pragma unroll
        for (int c = 0; c < VW; ++c) s[r][c] = fmaf(ki, u[c], s[r][c]);
    }
    if (state_out != nullptr) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < VW; ++c) state_out[sbase + (long)(row0 + r) * dv + col0 + c] = s[r][c];
    }
}

template <int DK, int DV>
cudaError_t launch_prologue_t(const PrologueArgs& a, cudaStream_t stream) {
    const dim3 grid((a.T + TT - 1) / TT, a.H, a.B);
    constexpr int threads = (2 * DK + DV) / 2;
    if (a.T > 0) {
        if (a.per_channel)
            prologue_kernel<DK, DV, true, TT><<<grid, threads, 0, stream>>>(
                a.q_raw, a.k_raw, a.v_raw, a.g_raw, a.beta_raw, a.conv_w, a.ring, a.pos0, a.silu,
                a.q, a.k, a.v, a.g, a.beta, a.T, a.H);
        else
            prologue_kernel<DK, DV, false, TT><<<grid, threads, 0, stream>>>(
                a.q_raw, a.k_raw, a.v_raw, a.g_raw, a.beta_raw, a.conv_w, a.ring, a.pos0, a.silu,
                a.q, a.k, a.v, a.g, a.beta, a.T, a.H);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.ring != nullptr && a.T > 0) {
        prologue_ring_kernel<DK, DV><<<a.B * a.H, 128, 0, stream>>>(a.q_raw, a.k_raw, a.v_raw, a.ring,
                                                                    a.pos0, a.T, a.H);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

constexpr int STEP_COLS = 64;   // value columns per CTA of the fused decode step
constexpr int STEP_WARPS = 4;

template <int DK, bool CHANNEL>
cudaError_t launch_step_t(const StepPrologueArgs& a, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(a.dv / STEP_COLS) * a.H * a.B;
    recurrent_prologue_kernel<DK, STEP_COLS, STEP_WARPS, CHANNEL><<<grid, STEP_WARPS * 32, 0, stream>>>(
        a.q_raw, a.k_raw, a.v_raw, a.g_raw, a.beta_raw, a.conv_w, a.ring, a.pos, a.silu, a.state_in,
        a.state_out, a.out, a.H, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
    if (a.dk == 128 && a.dv == 128) return launch_prologue_t<128, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_prologue_t<128, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_prologue_t<64, 128>(a, stream);
    if (a.dk == 64 && a.dv == 64) return launch_prologue_t<64, 64>(a, stream);
    return cudaErrorNotSupported;
}

cudaError_t launch_prologue_ring(const PrologueArgs& a, cudaStream_t stream) {
    if (a.ring == nullptr || a.T < 1) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128)
        prologue_ring_kernel<128, 128><<<a.B * a.H, 128, 0, stream>>>(a.q_raw, a.k_raw, a.v_raw, a.ring,
                                                                      a.pos0, a.T, a.H);
    else
        return cudaErrorNotSupported;
    return cudaGetLastError();
}

cudaError_t launch_step_prologue(const StepPrologueArgs& a, cudaStream_t stream) {
    if (a.dv % 64 != 0) return cudaErrorNotSupported;
    if (a.dk == 128) return a.per_channel ? launch_step_t<128, true>(a, stream) : launch_step_t<128, false>(a, stream);
    if (a.dk == 64) return a.per_channel ? launch_step_t<64, true>(a, stream) : launch_step_t<64, false>(a, stream);
    return cudaErrorNotSupported;
}

}  // namespace gdn
