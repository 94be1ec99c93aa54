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

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int TT = 32;   // tokens per CTA of the prefill prologue

__device__ __forceinline__ float act_fn(float y, bool silu) { return silu ? y / (1.f + expf(-y)) : y; }
__device__ __forceinline__ float sigmoid_fn(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float gate_fn(float x) {
    const float sp = x > 30.f ? x : log1pf(expf(x));
    return -fminf(sp, 5.f);
}

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

// One CTA: TT tokens of one (batch, head); one thread per pair of channels of
// q | k | v (CP = (2 dk + dv) / 2 threads).  Sliding window of the last three
// raw inputs in registers; the L2 norms of q and k through warp shuffles and
// one shared-memory exchange between the warps of a tensor.
template <int DK, int DV, bool CHANNEL>
__global__ void __launch_bounds__((2 * DK + DV) / 2)
prologue_kernel(const __nv_bfloat16* __restrict__ q_raw, const __nv_bfloat16* __restrict__ k_raw,
                const __nv_bfloat16* __restrict__ v_raw, const float* __restrict__ g_raw,
                const float* __restrict__ beta_raw, const float* __restrict__ conv_w,
                const float* __restrict__ ring, const int* __restrict__ pos0, bool silu,
                __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v,
                float* __restrict__ g, float* __restrict__ beta, int T, int H)
{
    constexpr int CH = 2 * DK + DV;
    constexpr int QW = DK / 64;                 // warps per q (and per k)
    __shared__ float s_ss[2][QW][TT];           // per-warp sums of squares, q and k

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = tile * TT;
    const int c = 2 * tid;                      // first channel of this thread
    const int p0 = pos0 ? pos0[b] : 0;

    const float* w = conv_w + ((long)h * CH + c) * 4;
    const float4 w0 = *reinterpret_cast<const float4*>(w);        // taps of channel c
    const float4 w1 = *reinterpret_cast<const float4*>(w + 4);    // taps of channel c + 1

    // Window: raw inputs at t0 - 3, t0 - 2, t0 - 1.
    float2 win[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int t = t0 - 3 + i;
        if (t >= 0) {
            win[i] = raw_pair(q_raw, k_raw, v_raw, ((long)b * T + t) * H + h, c, DK, DV);
        } else {
            const int p = p0 + t;
            win[i] = make_float2(0.f, 0.f);
            if (ring && p >= 0) {
                const float* r = ring + (((long)b * H + h) * 4 + (p & 3)) * CH + c;
                win[i] = make_float2(r[0], r[1]);
            }
        }
    }
    const int nt = min(TT, T - t0);
    float2 y[TT];
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        y[i] = make_float2(0.f, 0.f);
        if (i < nt) {
            const float2 x = raw_pair(q_raw, k_raw, v_raw, ((long)b * T + t0 + i) * H + h, c, DK, DV);
            float a0 = w0.x * win[0].x + w0.y * win[1].x + w0.z * win[2].x + w0.w * x.x;
            float a1 = w1.x * win[0].y + w1.y * win[1].y + w1.z * win[2].y + w1.w * x.y;
            y[i] = make_float2(act_fn(a0, silu), act_fn(a1, silu));
            win[0] = win[1]; win[1] = win[2]; win[2] = x;
        }
    }
    const int tensor = warp / QW;               // 0 q, 1 k, >= 2 v
    if (tensor < 2) {
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            float ss = y[i].x * y[i].x + y[i].y * y[i].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) s_ss[tensor][warp % QW][i] = ss;
        }
    }
    // beta and a scalar g: the v threads (which follow the DK threads of q and
    // k), one token each.
    if (tensor >= 2) {
        const int i = tid - DK;
        if (i < nt) {
            const long tok = ((long)b * T + t0 + i) * H + h;
            beta[tok] = sigmoid_fn(beta_raw[tok]);
            if (!CHANNEL) g[tok] = gate_fn(g_raw[tok]);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        if (i >= nt) break;
        const long tok = ((long)b * T + t0 + i) * H + h;
        float2 o = y[i];
        if (tensor < 2) {
            float ss = 0.f;
#pragma unroll
            for (int wq = 0; wq < QW; ++wq) ss += s_ss[tensor][wq][i];
            const float inv = rsqrtf(ss + 1e-6f);
            o.x *= inv; o.y *= inv;
        }
        const __nv_bfloat162 ob = __floats2bfloat162_rn(o.x, o.y);
        if (tensor == 0) {
            *reinterpret_cast<__nv_bfloat162*>(q + tok * DK + c) = ob;
            if (CHANNEL) {   // the q threads also map the per-channel gate
                const float2 gr = *reinterpret_cast<const float2*>(g_raw + tok * DK + c);
                *reinterpret_cast<float2*>(g + tok * DK + c) = make_float2(gate_fn(gr.x), gate_fn(gr.y));
            }
        } else if (tensor == 1) {
            *reinterpret_cast<__nv_bfloat162*>(k + tok * DK + (c - DK)) = ob;
        } else {
            *reinterpret_cast<__nv_bfloat162*>(v + tok * DV + (c - 2 * DK)) = ob;
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
__global__ void __launch_bounds__(NWARPS * 32)
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

    float s[R][VW];
    const long sbase = ((long)b * H + h) * DK * (long)dv;
    if (state_in != nullptr) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < VW; ++c) s[r][c] = state_in[sbase + (long)(row0 + r) * dv + col0 + c];
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < VW; ++c) s[r][c] = 0.f;
    }

    // Convolution of one channel: taps 0..2 from the ring, tap 3 the input.
    auto conv1 = [&](int ch, float x) -> float {
        const float4 w = *reinterpret_cast<const float4*>(conv_w + ((long)h * CH + ch) * 4);
        float hst[3] = {0.f, 0.f, 0.f};
        if (ring) {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int pp = p - 3 + j;
                if (pp >= 0) hst[j] = ring[(ring_bh + (pp & 3)) * CH + ch];
            }
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
    float sq = yq * yq, sk = yk * yk;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
    }
    if (lane == 0) { s_ss[0][warp] = sq; s_ss[1][warp] = sk; }
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
    {
        float nq = 0.f, nk = 0.f;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) { nq += s_ss[0][w]; nk += s_ss[1][w]; }
        if (tid < DK) {
            s_q[tid] = yq * rsqrtf(nq + 1e-6f);
            s_k[tid] = yk * rsqrtf(nk + 1e-6f);
        }
    }
    __syncthreads();

    // The decode step (as recurrent.cu): S' = Diag(a) S, x = S'^T k,
    // c = S'^T q, u = b (v - x), S = S' + k u^T, o = c + u (k . q).
    float px[VW], pc[VW];
#pragma unroll
    for (int c = 0; c < VW; ++c) { px[c] = 0.f; pc[c] = 0.f; }
    float kq = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float ki = s_k[row0 + r];
        const float qi = s_q[row0 + r];
        const float ai = CHANNEL ? s_a[row0 + r] : a_scalar;
        kq = fmaf(ki, qi, kq);
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
    if (lane == 0) s_kq[warp] = kq;
    __syncthreads();
    float kq_all = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) kq_all += s_kq[w];
    float u[VW];
#pragma unroll
    for (int c = 0; c < VW; ++c) {
        float x = 0.f, cc = 0.f;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) {
            x += s_red[0][w][lane * VW + c];
            cc += s_red[1][w][lane * VW + c];
        }
        u[c] = bt * (vv[c] - x);
        if (warp == 0) out[tok * dv + col0 + c] = fmaf(u[c], kq_all, cc);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float ki = s_k[row0 + r];
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
            prologue_kernel<DK, DV, true><<<grid, threads, 0, stream>>>(
                a.q_raw, a.k_raw, a.v_raw, a.g_raw, a.beta_raw, a.conv_w, a.ring, a.pos0, a.silu,
                a.q, a.k, a.v, a.g, a.beta, a.T, a.H);
        else
            prologue_kernel<DK, DV, false><<<grid, threads, 0, stream>>>(
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

template <int DK, bool CHANNEL>
cudaError_t launch_step_t(const StepPrologueArgs& a, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(a.dv / 64) * a.H * a.B;
    recurrent_prologue_kernel<DK, 64, 4, CHANNEL><<<grid, 128, 0, stream>>>(
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

cudaError_t launch_step_prologue(const StepPrologueArgs& a, cudaStream_t stream) {
    if (a.dv % 64 != 0) return cudaErrorNotSupported;
    if (a.dk == 128) return a.per_channel ? launch_step_t<128, true>(a, stream) : launch_step_t<128, false>(a, stream);
    if (a.dk == 64) return a.per_channel ? launch_step_t<64, true>(a, stream) : launch_step_t<64, false>(a, stream);
    return cudaErrorNotSupported;
}

}  // namespace gdn
