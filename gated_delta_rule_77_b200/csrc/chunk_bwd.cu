// chunk_bwd.cu -- gradients of the chunkwise Gated DeltaNet recurrence.
//
// Method: Atomic-GDN2 model card, section 2.1 ("Gated DeltaNet-2"), the
// recurrence S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t, a_t = exp(g_t); its chunkwise form is the one the
// training / prefill mode uses ("Gated DeltaNet" entity trail, finding of
// 2026-07-29).  Per chunk of C tokens with start state S, in-chunk cumulative
// gate G_r (inclusive; a dk-vector per token, or a scalar), E_r = exp(G_r):
//
//   Abar_rj = k_r^T Diag(exp(G_r - G_j)) k_j  (j < r),  A = Diag(b) Abar,
//   T = (I + A)^-1,  P_rj = q_r^T Diag(exp(G_r - G_j)) k_j  (j <= r),
//   Kt = E (.) K,  Qt = E (.) Q,  Kh_j = exp(G_last - G_j) (.) k_j,
//   X = Diag(b)(V - Kt S),  U = T X,  O = Qt S + P U,
//   S_next = Diag(E_last) S + Kh^T U.
//
// Reverse mode through that chunk, given dO and dS_next (the gradient of the
// chunk's end state), derived from the forward above by the chain rule:
//
//   dU  = Kh dS_next + P^T dO,   Y = T^T dU,   dV = Diag(b) Y
//   G   = -strictlower(Y U^T),   dP = lower(dO U^T)
//   db_r = Y_r . (V - Kt S)_r + sum_j G_rj Abar_rj
//   dS  = Diag(E_last) dS_next + Qt^T dO - Kt^T Diag(b) Y      (the chain)
//   dQt = dO S^T,  dKt = -Diag(b) Y S^T,  dKh = U dS_next^T
//   dQ  = E (.) dQt + [sum_j dP_rj decay(r,j) (.) k_j]
//   dK  = E (.) dKt + exp(G_last - G) (.) dKh + [row and column roles of
//         the decay-weighted products of A and P]
//   dG_r = Qt (.) dQt + Kt (.) dKt - Kh (.) dKh + (row role - column role of
//         A and P) ;  dG_last += E_last (.) rowsum(dS_next (.) S) + sum_j Kh_j (.) dKh_j
//   dg_s = sum_{r >= s} dG_r  (within the chunk; summed over channels for a
//          scalar gate)
//
// Chunk of C = 32 tokens.  A per-channel gate (g >= -5) is handled with one
// reference token m = 16 per chunk: exp(G_r - G_j) = L_r R_j with
// L = exp(G - G_m), R = exp(G_m - G), both within e^{+-80} (fp32 range) for
// |r - m| <= 16 -- the model card's bound 160 / bs2 with bs2 = 32.  The
// decay-weighted products then become plain products of (L (.) K), (R (.) K),
// (L (.) Q).  A scalar gate (any g <= 0) uses the exact C x C ratio matrix.
//
// Passes (all fp32 arithmetic on bf16 / fp32 inputs, CUDA cores):
//   1. bwd_prep_kernel      per chunk: T, W = T Diag(b) Kt, Ut = T Diag(b) V,
//                           Kh, Qt, P, E_last -> scratch;
//   2. bwd_state_chain      per (b, h, 32-column slice), forward over chunks:
//                           S_next = Diag(E_last) S + Kh^T (Ut - W S); stores
//                           every chunk's start state;
//   3. bwd_dstate_chain     per (b, h, slice), backward over chunks:
//                           dS = Diag(E_last) dS_next + Qt^T dO
//                                - W^T (Kh dS_next + P^T dO); stores every
//                           chunk's dS_next; the last one is d(state_in);
//   4. bwd_grads_kernel     per chunk: everything else above.

#include <math.h>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int BC = 32;          // chunk length
constexpr int BM = 16;          // reference token of the per-channel decay
constexpr int BNT = 256;        // threads per CTA
constexpr int CP = BC + 1;      // padded row length of a C x C matrix

// out(r, c) for r < 32, c < N: warp w owns rows 4w .. 4w+3, lane l the
// columns l, l + 32, ..., so that a row-major B operand is read by
// consecutive lanes and a transposed one (row stride = 1 mod 32) without
// bank conflicts; the A operand is one address per warp (a broadcast).
template <int N, int K, typename FA, typename FB>
__device__ __forceinline__ void mm32(float (&acc)[4][N / 32], FA a, FB b) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float av[4], bv[N / 32];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = a(4 * w + i, kk);
#pragma unroll
        for (int j = 0; j < N / 32; ++j) bv[j] = b(kk, l + 32 * j);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < N / 32; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

template <int N>
__device__ __forceinline__ void zero4(float (&acc)[4][N]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) acc[i][j] = 0.f;
}

// Scratch of one (b, h, chunk) for the chains (fp32): W, Kh, Qt [C][DK],
// Ut [C][DV], P [C][C], E_last [DK].
template <int DK, int DV>
struct ChunkScratch {
    static constexpr long kW = 0;
    static constexpr long kKh = kW + BC * DK;
    static constexpr long kQt = kKh + BC * DK;
    static constexpr long kUt = kQt + BC * DK;
    static constexpr long kP = kUt + BC * DV;
    static constexpr long kEl = kP + BC * BC;
    static constexpr long kSize = kEl + DK;
};

// Shared-memory tiles of the chunk-local part common to the prep and the
// gradient kernels.
template <int DK, int CHANNEL>
struct Local {
    static constexpr int KP = DK + 1;            // padded row of a C x DK tile
    float KL[BC][KP];      // channel: L (.) K ; scalar: K
    float KR[BC][KP];      // channel: R (.) K ; scalar: K
    float QL[BC][KP];      // channel: L (.) Q ; scalar: Q
    float Gam[BC][CHANNEL ? DK : 1];   // in-chunk cumulative gate
    float Abar[BC][CP];    // strictly lower; decay applied
    float Tm[BC][CP];      // (I + A)^-1
    float P[BC][CP];       // lower incl. diagonal; decay applied
    float D[CHANNEL ? 1 : BC][CHANNEL ? 1 : CP];   // scalar gate: exp(G_r - G_j), j <= r
    float beta[BC];
    float Gm[CHANNEL ? DK : 1];       // G at the reference token
    float Gl[CHANNEL ? DK : 1];       // G at the last token
};

// Loads one chunk (zero past T: k = q = 0, g = 0, beta = 0 leave the state
// unchanged), forms the cumulative gate, the decay factors, Abar, P and T.
template <int DK, int CHANNEL>
__device__ void chunk_local(Local<DK, CHANNEL>& s, const __nv_bfloat16* __restrict__ q,
                            const __nv_bfloat16* __restrict__ k, const float* __restrict__ g,
                            const float* __restrict__ beta, int b, int h, int t0, int T, int H)
{
    const int tid = threadIdx.x;
    for (int idx = tid; idx < BC * DK; idx += BNT) {
        const int r = idx / DK, c = idx % DK;
        const int t = t0 + r;
        float kv = 0.f, qv = 0.f;
        if (t < T) {
            const long tok = ((long)b * T + t) * H + h;
            kv = __bfloat162float(k[tok * DK + c]);
            qv = __bfloat162float(q[tok * DK + c]);
            if (CHANNEL) s.Gam[r][c] = g[tok * DK + c];
        } else if (CHANNEL) {
            s.Gam[r][c] = 0.f;
        }
        s.KL[r][c] = kv;
        s.QL[r][c] = qv;
    }
    if (tid < BC) {
        const int t = t0 + tid;
        const long tok = ((long)b * T + t) * H + h;
        s.beta[tid] = t < T ? beta[tok] : 0.f;
        if (!CHANNEL) s.Gam[tid][0] = t < T ? g[tok] : 0.f;
    }
    __syncthreads();
    // Inclusive cumulative sum over the chunk, one channel per thread.
    constexpr int NCH = CHANNEL ? DK : 1;
    for (int c = tid; c < NCH; c += BNT) {
        float acc = 0.f;
#pragma unroll 8
        for (int r = 0; r < BC; ++r) {
            acc += s.Gam[r][c];
            s.Gam[r][c] = acc;
        }
        s.Gm[c] = s.Gam[BM][c];
        s.Gl[c] = acc;
    }
    __syncthreads();
    if (CHANNEL) {
        for (int idx = tid; idx < BC * DK; idx += BNT) {
            const int r = idx / DK, c = idx % DK;
            const float d = s.Gam[r][c] - s.Gm[c];
            const float L = expf(d), R = expf(-d);
            const float kv = s.KL[r][c];
            s.KR[r][c] = kv * R;
            s.KL[r][c] = kv * L;
            s.QL[r][c] *= L;
        }
    } else {
        for (int idx = tid; idx < BC * DK; idx += BNT) {
            const int r = idx / DK, c = idx % DK;
            s.KR[r][c] = s.KL[r][c];
        }
        for (int idx = tid; idx < BC * BC; idx += BNT) {
            const int r = idx / BC, j = idx % BC;
            s.D[r][j] = j <= r ? expf(s.Gam[r][0] - s.Gam[j][0]) : 0.f;
        }
    }
    __syncthreads();
    // Abar = KL KR^T (strictly lower), P = QL KR^T (lower), decay applied.
    {
        float aa[4][1], pp[4][1];
        zero4(aa);
        zero4(pp);
        mm32<BC, DK>(aa, [&](int r, int kk) { return s.KL[r][kk]; },
                     [&](int kk, int j) { return s.KR[j][kk]; });
        mm32<BC, DK>(pp, [&](int r, int kk) { return s.QL[r][kk]; },
                     [&](int kk, int j) { return s.KR[j][kk]; });
        const int w = tid >> 5, j = tid & 31;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * w + i;
            const float dec = CHANNEL ? 1.f : s.D[r][j];
            s.Abar[r][j] = j < r ? aa[i][0] * dec : 0.f;
            s.P[r][j] = j <= r ? pp[i][0] * dec : 0.f;
        }
    }
    __syncthreads();
    // T = (I + Diag(beta) Abar)^-1 by forward substitution: lane j of warp 0
    // solves column j.
    if (tid < 32) {
        const int j = tid;
        float x[BC];
#pragma unroll
        for (int i = 0; i < BC; ++i) {
            float v = i == j ? 1.f : 0.f;
            const float bi = s.beta[i];
#pragma unroll
            for (int l = 0; l < i; ++l) v = fmaf(-bi * s.Abar[i][l], x[l], v);
            x[i] = v;
        }
#pragma unroll
        for (int i = 0; i < BC; ++i) s.Tm[i][j] = x[i];
    }
    __syncthreads();
}

// Pass 1: the chain's per-chunk operands.  grid (chunks, H, B).
template <int DK, int DV, int CHANNEL>
__global__ void __launch_bounds__(BNT)
bwd_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                const float* __restrict__ beta, float* __restrict__ scratch, int T, int H, int N)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    using L = Local<DK, CHANNEL>;
    using SC = ChunkScratch<DK, DV>;
    L& s = *reinterpret_cast<L*>(smem_raw);
    float (*sV)[DV + 1] = reinterpret_cast<float (*)[DV + 1]>(smem_raw + sizeof(L));
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * BC, tid = threadIdx.x;
    for (int idx = tid; idx < BC * DV; idx += BNT) {
        const int r = idx / DV, j = idx % DV;
        const int t = t0 + r;
        sV[r][j] = t < T ? __bfloat162float(v[(((long)b * T + t) * H + h) * DV + j]) : 0.f;
    }
    chunk_local<DK, CHANNEL>(s, q, k, g, beta, b, h, t0, T, H);
    float* out = scratch + (((long)b * H + h) * N + c) * SC::kSize;

    // Kt = E (.) K and Qt = E (.) Q, Kh = exp(G_last - G) (.) K.
    auto e_of = [&](int r, int cc) -> float {   // E_rc = exp(G_rc)
        return CHANNEL ? expf(s.Gam[r][cc]) : expf(s.Gam[r][0]);
    };
    const int w = tid >> 5, l = tid & 31;
    {
        float acc[4][DK / 32];
        zero4(acc);
        if (CHANNEL) {
            mm32<DK, BC>(acc, [&](int r, int j) { return s.Tm[r][j] * s.beta[j]; },
                         [&](int j, int cc) { return s.KL[j][cc]; });
        } else {
            mm32<DK, BC>(acc, [&](int r, int j) { return s.Tm[r][j] * s.beta[j] * expf(s.Gam[j][0]); },
                         [&](int j, int cc) { return s.KL[j][cc]; });
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < DK / 32; ++jj) {
                const int r = 4 * w + i, cc = l + 32 * jj;
                // channel: W = T Diag(b) (L (.) K) scaled by E_m per channel
                out[SC::kW + r * DK + cc] = CHANNEL ? acc[i][jj] * expf(s.Gm[cc]) : acc[i][jj];
            }
    }
    {
        float acc[4][DV / 32];
        zero4(acc);
        mm32<DV, BC>(acc, [&](int r, int j) { return s.Tm[r][j] * s.beta[j]; },
                     [&](int j, int cc) { return sV[j][cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < DV / 32; ++jj) out[SC::kUt + (4 * w + i) * DV + l + 32 * jj] = acc[i][jj];
    }
    for (int idx = tid; idx < BC * DK; idx += BNT) {
        const int r = idx / DK, cc = idx % DK;
        float kh, qt;
        if (CHANNEL) {
            kh = s.KR[r][cc] * expf(s.Gl[cc] - s.Gm[cc]);
            qt = s.QL[r][cc] * expf(s.Gm[cc]);
        } else {
            kh = s.KL[r][cc] * expf(s.Gl[0] - s.Gam[r][0]);
            qt = s.QL[r][cc] * e_of(r, cc);
        }
        out[SC::kKh + idx] = kh;
        out[SC::kQt + idx] = qt;
    }
    for (int idx = tid; idx < BC * BC; idx += BNT) out[SC::kP + idx] = s.P[idx / BC][idx % BC];
    for (int cc = tid; cc < DK; cc += BNT) out[SC::kEl + cc] = expf(CHANNEL ? s.Gl[cc] : s.Gl[0]);
}

// Shared memory of the two chains (per 32-column slice of the state).
template <int DK>
struct ChainSmem {
    float W[BC][DK + 1];
    float Kh[BC][DK + 1];
    float Qt[BC][DK + 1];
    float P[BC][CP];
    float dO[BC][33];
    float Z[BC][33];
    float S[DK][33];
    float El[DK];
};

// Pass 2: chunk start states, forward over the chunks of one (b, h) for a
// slice of 32 value columns.  grid (DV / 32, H, B).
template <int DK, int DV>
__global__ void __launch_bounds__(BNT)
bwd_state_chain_kernel(const float* __restrict__ scratch, const float* __restrict__ state_in,
                       float* __restrict__ states, int H, int N)
{
    using SC = ChunkScratch<DK, DV>;
    constexpr int RW = DK / 8;                     // state rows per warp
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ChainSmem<DK>& cs = *reinterpret_cast<ChainSmem<DK>*>(smem_raw);
    auto& sW = cs.W;
    auto& sKh = cs.Kh;
    auto& sZ = cs.Z;
    auto& sS = cs.S;
    auto& sEl = cs.El;
    const int sl = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int col = sl * 32 + l;
    const long bh = (long)b * H + h;
    float st[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i)
        st[i] = state_in ? state_in[(bh * DK + RW * w + i) * DV + col] : 0.f;
    for (int c = 0; c < N; ++c) {
        const float* src = scratch + (bh * N + c) * SC::kSize;
        float* dst = states + ((bh * N + c) * DK) * (long)DV;
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            dst[(long)(RW * w + i) * DV + col] = st[i];
            sS[RW * w + i][l] = st[i];
        }
        for (int idx = tid; idx < BC * DK; idx += BNT) {
            sW[idx / DK][idx % DK] = src[SC::kW + idx];
            sKh[idx / DK][idx % DK] = src[SC::kKh + idx];
        }
        for (int cc = tid; cc < DK; cc += BNT) sEl[cc] = src[SC::kEl + cc];
        __syncthreads();
        // Z = Ut - W S  (C x 32)
        float z[4][1];
        zero4(z);
        mm32<32, DK>(z, [&](int r, int kk) { return sW[r][kk]; }, [&](int kk, int j) { return sS[kk][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
            sZ[4 * w + i][l] = src[SC::kUt + (4 * w + i) * DV + col] - z[i][0];
        __syncthreads();
        // S = Diag(E_last) S + Kh^T Z
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            const int r = RW * w + i;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < BC; ++j) acc = fmaf(sKh[j][r], sZ[j][l], acc);
            st[i] = fmaf(sEl[r], st[i], acc);
        }
        __syncthreads();
    }
}

// Pass 3: dS at every chunk end, backward over the chunks of one (b, h) for
// a slice of 32 value columns; writes d(state_in).  grid (DV / 32, H, B).
template <int DK, int DV>
__global__ void __launch_bounds__(BNT)
bwd_dstate_chain_kernel(const float* __restrict__ scratch, const float* __restrict__ d_out,
                        const float* __restrict__ d_state_out, float* __restrict__ dstates,
                        float* __restrict__ d_state_in, int T, int H, int N)
{
    using SC = ChunkScratch<DK, DV>;
    constexpr int RW = DK / 8;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ChainSmem<DK>& cs = *reinterpret_cast<ChainSmem<DK>*>(smem_raw);
    auto& sW = cs.W;
    auto& sKh = cs.Kh;
    auto& sQt = cs.Qt;
    auto& sP = cs.P;
    auto& sdO = cs.dO;
    auto& sZ = cs.Z;
    auto& sS = cs.S;
    auto& sEl = cs.El;
    const int sl = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int col = sl * 32 + l;
    const long bh = (long)b * H + h;
    float ds[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i)
        ds[i] = d_state_out ? d_state_out[(bh * DK + RW * w + i) * DV + col] : 0.f;
    for (int c = N - 1; c >= 0; --c) {
        const float* src = scratch + (bh * N + c) * SC::kSize;
        float* dst = dstates + ((bh * N + c) * DK) * (long)DV;
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            dst[(long)(RW * w + i) * DV + col] = ds[i];
            sS[RW * w + i][l] = ds[i];
        }
        for (int idx = tid; idx < BC * DK; idx += BNT) {
            sW[idx / DK][idx % DK] = src[SC::kW + idx];
            sKh[idx / DK][idx % DK] = src[SC::kKh + idx];
            sQt[idx / DK][idx % DK] = src[SC::kQt + idx];
        }
        for (int idx = tid; idx < BC * BC; idx += BNT) sP[idx / BC][idx % BC] = src[SC::kP + idx];
        for (int cc = tid; cc < DK; cc += BNT) sEl[cc] = src[SC::kEl + cc];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = c * BC + 4 * w + i;
            sdO[4 * w + i][l] = t < T ? d_out[(((long)b * T + t) * H + h) * DV + col] : 0.f;
        }
        __syncthreads();
        // Z = Kh dS_next + P^T dO  (C x 32)
        float z[4][1];
        zero4(z);
        mm32<32, DK>(z, [&](int r, int kk) { return sKh[r][kk]; }, [&](int kk, int j) { return sS[kk][j]; });
        mm32<32, BC>(z, [&](int r, int j) { return sP[j][r]; }, [&](int j, int cc) { return sdO[j][cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i) sZ[4 * w + i][l] = z[i][0];
        __syncthreads();
        // dS = Diag(E_last) dS_next + Qt^T dO - W^T Z
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            const int r = RW * w + i;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < BC; ++j) acc = fmaf(sQt[j][r], sdO[j][l], fmaf(-sW[j][r], sZ[j][l], acc));
            ds[i] = fmaf(sEl[r], ds[i], acc);
        }
        __syncthreads();
    }
    if (d_state_in) {
#pragma unroll
        for (int i = 0; i < RW; ++i) d_state_in[(bh * DK + RW * w + i) * DV + col] = ds[i];
    }
}

// Shared memory of the gradient kernel beyond the chunk-local tiles.
template <int DK, int DV, int CHANNEL>
struct GradSmem {
    Local<DK, CHANNEL> loc;
    float V[BC][DV + 1];       // v, then E2 = V - Kt S
    float dO[BC][DV + 1];      // dO, then dU, then Y
    float U[BC][DV + 1];
    float Big[DK][DV + 1];     // S, dS_next, S again, then dG [C][DK]
    float dP[BC][CP];          // lower(dO U^T), no decay
    float Gm2[BC][CP];         // -strictlower(Y U^T), no decay
    float rowdot[DK];          // rowsum(dS_next (.) S)
    float last[8][DK];         // per-warp column sums of Kh (.) dKh
    float db[BC];
    float eM[CHANNEL ? DK : BC];    // channel: exp(G_m); scalar: E_r = exp(G_r)
    float eH[CHANNEL ? DK : BC];    // channel: exp(G_last - G_m); scalar: exp(G_last - G_r)
};

// Pass 4: gradients of one chunk's tokens.  grid (chunks, H, B).
template <int DK, int DV, int CHANNEL>
__global__ void __launch_bounds__(BNT)
bwd_grads_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ beta, const float* __restrict__ d_out,
                 const float* __restrict__ states, const float* __restrict__ dstates,
                 float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                 float* __restrict__ dg, float* __restrict__ dbeta, int T, int H, int N)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    using SM = GradSmem<DK, DV, CHANNEL>;
    SM& m = *reinterpret_cast<SM*>(smem_raw);
    auto& s = m.loc;
    constexpr int NK = DK / 32, NV = DV / 32;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * BC, tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const long n = ((long)b * H + h) * N + c;
    const float* gS = states + n * DK * (long)DV;
    const float* gdS = dstates + n * DK * (long)DV;
    auto tok_of = [&](int r) -> long { return ((long)b * T + t0 + r) * H + h; };

    for (int idx = tid; idx < BC * DV; idx += BNT) {
        const int r = idx / DV, j = idx % DV;
        const bool in = t0 + r < T;
        m.V[r][j] = in ? __bfloat162float(v[tok_of(r) * DV + j]) : 0.f;
        m.dO[r][j] = in ? d_out[tok_of(r) * DV + j] : 0.f;
    }
    for (int idx = tid; idx < DK * DV; idx += BNT) m.Big[idx / DV][idx % DV] = gS[idx];
    chunk_local<DK, CHANNEL>(s, q, k, g, beta, b, h, t0, T, H);   // ends with a barrier
    if (CHANNEL) {
        for (int cc = tid; cc < DK; cc += BNT) {
            m.eM[cc] = expf(s.Gm[cc]);
            m.eH[cc] = expf(s.Gl[cc] - s.Gm[cc]);
        }
    } else if (tid < BC) {
        m.eM[tid] = expf(s.Gam[tid][0]);
        m.eH[tid] = expf(s.Gl[0] - s.Gam[tid][0]);
    }
    __syncthreads();

    // Per-element factors of this thread's outputs (rows 4w + i, columns
    // l + 32 jj of a C x DK tile).
    auto Kt = [&](int r, int cc) { return CHANNEL ? s.KL[r][cc] * m.eM[cc] : s.KL[r][cc] * m.eM[r]; };
    auto Qt = [&](int r, int cc) { return CHANNEL ? s.QL[r][cc] * m.eM[cc] : s.QL[r][cc] * m.eM[r]; };
    auto Kh = [&](int r, int cc) { return CHANNEL ? s.KR[r][cc] * m.eH[cc] : s.KL[r][cc] * m.eH[r]; };
    auto Eo = [&](int r, int cc) { return CHANNEL ? expf(s.Gam[r][cc]) : m.eM[r]; };
    auto Eho = [&](int r, int cc) { return CHANNEL ? expf(s.Gl[cc] - s.Gam[r][cc]) : m.eH[r]; };

    float dQa[4][NK], dKa[4][NK], dGa[4][NK];
    zero4(dQa);
    zero4(dKa);
    zero4(dGa);

    // E2 = V - Kt S (in place in V); dQt = dO S^T.
    {
        float acc[4][NV];
        zero4(acc);
        mm32<DV, DK>(acc, Kt, [&](int kk, int j) { return m.Big[kk][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) m.V[4 * w + i][l + 32 * jj] -= acc[i][jj];
    }
    {
        float acc[4][NK];
        zero4(acc);
        mm32<DK, DV>(acc, [&](int r, int j) { return m.dO[r][j]; }, [&](int j, int cc) { return m.Big[cc][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                const int r = 4 * w + i, cc = l + 32 * jj;
                dQa[i][jj] += Eo(r, cc) * acc[i][jj];
                dGa[i][jj] += Qt(r, cc) * acc[i][jj];
            }
    }
    __syncthreads();
    // U = T Diag(b) E2.
    {
        float acc[4][NV];
        zero4(acc);
        mm32<DV, BC>(acc, [&](int r, int j) { return s.Tm[r][j] * s.beta[j]; },
                     [&](int j, int cc) { return m.V[j][cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) m.U[4 * w + i][l + 32 * jj] = acc[i][jj];
    }
    // rowsum(dS_next (.) S), one row per warp at a time.
    for (int r = w; r < DK; r += 8) {
        float acc = 0.f;
        for (int j = l; j < DV; j += 32) acc = fmaf(gdS[(long)r * DV + j], m.Big[r][j], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (l == 0) m.rowdot[r] = acc;
    }
    __syncthreads();
    // dP = lower(dO U^T); dS_next replaces S.
    {
        float acc[4][1];
        zero4(acc);
        mm32<BC, DV>(acc, [&](int r, int j) { return m.dO[r][j]; }, [&](int j, int jj) { return m.U[jj][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i) m.dP[4 * w + i][l] = l <= 4 * w + i ? acc[i][0] : 0.f;
    }
    for (int idx = tid; idx < DK * DV; idx += BNT) m.Big[idx / DV][idx % DV] = gdS[idx];
    __syncthreads();
    // dKh = U dS_next^T.
    {
        float acc[4][NK];
        zero4(acc);
        mm32<DK, DV>(acc, [&](int r, int j) { return m.U[r][j]; }, [&](int j, int cc) { return m.Big[cc][j]; });
#pragma unroll
        for (int jj = 0; jj < NK; ++jj) {
            const int cc = l + 32 * jj;
            float colsum = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 4 * w + i;
                const float kh = Kh(r, cc);
                dKa[i][jj] += Eho(r, cc) * acc[i][jj];
                dGa[i][jj] -= kh * acc[i][jj];
                colsum = fmaf(kh, acc[i][jj], colsum);
            }
            m.last[w][cc] = colsum;
        }
    }
    // dU = Kh dS_next + P^T dO (into dO once every thread is done with dO).
    {
        float acc[4][NV];
        zero4(acc);
        mm32<DV, DK>(acc, Kh, [&](int kk, int j) { return m.Big[kk][j]; });
        mm32<DV, BC>(acc, [&](int r, int j) { return s.P[j][r]; }, [&](int j, int cc) { return m.dO[j][cc]; });
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) m.dO[4 * w + i][l + 32 * jj] = acc[i][jj];
        __syncthreads();
    }
    // Y = T^T dU (into dO).
    {
        float acc[4][NV];
        zero4(acc);
        mm32<DV, BC>(acc, [&](int r, int j) { return s.Tm[j][r]; }, [&](int j, int cc) { return m.dO[j][cc]; });
        __syncthreads();
        float dbp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * w + i;
#pragma unroll
            for (int jj = 0; jj < NV; ++jj) {
                const int cc = l + 32 * jj;
                m.dO[r][cc] = acc[i][jj];
                dbp[i] = fmaf(acc[i][jj], m.V[r][cc], dbp[i]);
                if (t0 + r < T) dv[tok_of(r) * DV + cc] = s.beta[r] * acc[i][jj];
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dbp[i] += __shfl_xor_sync(0xffffffffu, dbp[i], o);
            if (l == 0) m.db[4 * w + i] = dbp[i];
        }
        __syncthreads();
    }
    // G = -strictlower(Y U^T); db += rowsum(G (.) Abar).  S replaces dS_next.
    {
        float acc[4][1];
        zero4(acc);
        mm32<BC, DV>(acc, [&](int r, int j) { return m.dO[r][j]; }, [&](int j, int jj) { return m.U[jj][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * w + i;
            const float gv = l < r ? -acc[i][0] : 0.f;
            m.Gm2[r][l] = gv;
            float x = gv * s.Abar[r][l];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (l == 0) m.db[r] += x;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < DK * DV; idx += BNT) m.Big[idx / DV][idx % DV] = gS[idx];
    __syncthreads();
    // dKt = -Diag(b) Y S^T.
    {
        float acc[4][NK];
        zero4(acc);
        mm32<DK, DV>(acc, [&](int r, int j) { return -s.beta[r] * m.dO[r][j]; },
                     [&](int j, int cc) { return m.Big[cc][j]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                const int r = 4 * w + i, cc = l + 32 * jj;
                dKa[i][jj] += Eo(r, cc) * acc[i][jj];
                dGa[i][jj] += Kt(r, cc) * acc[i][jj];
            }
    }
    // The decay-weighted products of A and P: rows and columns.
    auto decay = [&](int r, int j) { return CHANNEL ? 1.f : s.D[r][j]; };
    auto Lf = [&](int r, int cc) { return expf(s.Gam[r][cc] - s.Gm[cc]); };
    {   // t_row = (b G) KR ; t_col = (b G)^T KL
        float tr[4][NK], tc[4][NK];
        zero4(tr);
        zero4(tc);
        mm32<DK, BC>(tr, [&](int r, int j) { return s.beta[r] * m.Gm2[r][j] * decay(r, j); },
                     [&](int j, int cc) { return s.KR[j][cc]; });
        mm32<DK, BC>(tc, [&](int r, int j) { return s.beta[j] * m.Gm2[j][r] * decay(j, r); },
                     [&](int j, int cc) { return s.KL[j][cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                const int r = 4 * w + i, cc = l + 32 * jj;
                if (CHANNEL) {
                    const float L = Lf(r, cc), R = 1.f / L;
                    dKa[i][jj] += L * tr[i][jj] + R * tc[i][jj];
                    dGa[i][jj] += s.KL[r][cc] * tr[i][jj] - s.KR[r][cc] * tc[i][jj];
                } else {
                    dKa[i][jj] += tr[i][jj] + tc[i][jj];
                }
            }
    }
    {   // p_row = dP KR ; p_col = dP^T QL
        float pr[4][NK], pc[4][NK];
        zero4(pr);
        zero4(pc);
        mm32<DK, BC>(pr, [&](int r, int j) { return m.dP[r][j] * decay(r, j); },
                     [&](int j, int cc) { return s.KR[j][cc]; });
        mm32<DK, BC>(pc, [&](int r, int j) { return m.dP[j][r] * decay(j, r); },
                     [&](int j, int cc) { return s.QL[j][cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                const int r = 4 * w + i, cc = l + 32 * jj;
                if (CHANNEL) {
                    const float L = Lf(r, cc), R = 1.f / L;
                    dQa[i][jj] += L * pr[i][jj];
                    dKa[i][jj] += R * pc[i][jj];
                    dGa[i][jj] += s.QL[r][cc] * pr[i][jj] - s.KR[r][cc] * pc[i][jj];
                } else {
                    dQa[i][jj] += pr[i][jj];
                    dKa[i][jj] += pc[i][jj];
                }
            }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 4 * w + i;
        if (t0 + r < T) {
#pragma unroll
            for (int jj = 0; jj < NK; ++jj) {
                dq[tok_of(r) * DK + l + 32 * jj] = dQa[i][jj];
                dk[tok_of(r) * DK + l + 32 * jj] = dKa[i][jj];
            }
        }
    }
    __syncthreads();   // every read of Big (S) is done
    // dG per token and channel, then the reverse in-chunk cumulative sum.
    float* sdG = &m.Big[0][0];               // [C][DK]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < NK; ++jj) sdG[(4 * w + i) * DK + l + 32 * jj] = dGa[i][jj];
    __syncthreads();
    if (CHANNEL) {
        for (int cc = tid; cc < DK; cc += BNT) {
            float lastc = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) lastc += m.last[ww][cc];
            float acc = expf(s.Gl[cc]) * m.rowdot[cc] + lastc;   // at the last token
            for (int r = BC - 1; r >= 0; --r) {
                acc += sdG[r * DK + cc];
                if (t0 + r < T) dg[tok_of(r) * DK + cc] = acc;
            }
        }
    } else {
        // Scalar gate: the channel sums of the per-element terms, the row and
        // column sums of (b G) (.) Abar and dP (.) P, and the last-token term.
        float* rowv = &m.last[0][0];            // reuse: [C] after the sums below
        __shared__ float s_lastsum;
        if (w == 0) {
            float x = 0.f;
            for (int cc = l; cc < DK; cc += 32) {
                float lastc = 0.f;
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) lastc += m.last[ww][cc];
                x += expf(s.Gl[0]) * m.rowdot[cc] + lastc;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (l == 0) s_lastsum = x;
        }
        __syncthreads();
        // One warp per 4 rows: per-element channel sums and the C x C terms.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * w + i;
            float x = 0.f;
            for (int cc = l; cc < DK; cc += 32) x += sdG[r * DK + cc];
            const float ga = s.beta[r] * m.Gm2[r][l] * s.Abar[r][l] + m.dP[r][l] * s.P[r][l];
            const float gb = s.beta[l] * m.Gm2[l][r] * s.Abar[l][r] + m.dP[l][r] * s.P[l][r];
            x += ga - gb;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (l == 0) rowv[r] = x;
        }
        __syncthreads();
        if (tid == 0) {
            float acc = s_lastsum;
            for (int r = BC - 1; r >= 0; --r) {
                acc += rowv[r];
                if (t0 + r < T) dg[tok_of(r)] = acc;
            }
        }
    }
    if (tid < BC && t0 + tid < T) dbeta[tok_of(tid)] = m.db[tid];
}

template <int DK, int DV, int CHANNEL>
cudaError_t launch_bwd_t(const BwdProblem& p, cudaStream_t stream) {
    using SC = ChunkScratch<DK, DV>;
    const int N = (p.T + BC - 1) / BC;
    const long nchunks = (long)p.B * p.H * N;
    const size_t chunk_bytes = (size_t)nchunks * SC::kSize * sizeof(float);
    const size_t state_bytes = (size_t)nchunks * DK * DV * sizeof(float);
    float* ws = nullptr;
    cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&ws), chunk_bytes + 2 * state_bytes, stream);
    if (e != cudaSuccess) return e;
    float* scratch = ws;
    float* states = ws + nchunks * SC::kSize;
    float* dstates = states + nchunks * (long)DK * DV;
    const dim3 grid_c(N, p.H, p.B), grid_s(DV / 32, p.H, p.B);
    const size_t prep_smem = sizeof(Local<DK, CHANNEL>) + sizeof(float) * BC * (DV + 1);
    const size_t grad_smem = sizeof(GradSmem<DK, DV, CHANNEL>);
    const size_t chain_smem = sizeof(ChainSmem<DK>);
    static_assert(sizeof(GradSmem<DK, DV, CHANNEL>) <= 227 * 1024, "gradient tiles exceed shared memory");
    static_assert(sizeof(Local<DK, CHANNEL>) + sizeof(float) * BC * (DV + 1) <= 227 * 1024, "prep tiles");
    auto kp = bwd_prep_kernel<DK, DV, CHANNEL>;
    auto kg = bwd_grads_kernel<DK, DV, CHANNEL>;
    auto ks = bwd_state_chain_kernel<DK, DV>;
    auto kd = bwd_dstate_chain_kernel<DK, DV>;
    e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grad_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem);
    if (e == cudaSuccess) {
        kp<<<grid_c, BNT, prep_smem, stream>>>(p.q, p.k, p.v, p.g, p.beta, scratch, p.T, p.H, N);
        ks<<<grid_s, BNT, chain_smem, stream>>>(scratch, p.state_in, states, p.H, N);
        kd<<<grid_s, BNT, chain_smem, stream>>>(scratch, p.d_out, p.d_state_out, dstates, p.d_state_in,
                                                p.T, p.H, N);
        kg<<<grid_c, BNT, grad_smem, stream>>>(p.q, p.k, p.v, p.g, p.beta, p.d_out, states, dstates,
                                               p.dq, p.dk, p.dv, p.dg, p.dbeta, p.T, p.H, N);
        e = cudaGetLastError();
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : ef;
}

template <int DK, int DV>
cudaError_t launch_bwd_dims(const BwdProblem& p, cudaStream_t stream) {
    return p.per_channel ? launch_bwd_t<DK, DV, 1>(p, stream) : launch_bwd_t<DK, DV, 0>(p, stream);
}

}  // namespace

cudaError_t launch_chunk_bwd(const BwdProblem& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    if (p.Dk == 128 && p.Dv == 128) return launch_bwd_dims<128, 128>(p, stream);
    if (p.Dk == 128 && p.Dv == 64) return launch_bwd_dims<128, 64>(p, stream);
    if (p.Dk == 64 && p.Dv == 128) return launch_bwd_dims<64, 128>(p, stream);
    if (p.Dk == 64 && p.Dv == 64) return launch_bwd_dims<64, 64>(p, stream);
    return cudaErrorNotSupported;
}

}  // namespace gdn
