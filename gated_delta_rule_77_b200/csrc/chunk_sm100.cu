// chunk_sm100.cu -- chunkwise-parallel prefill of the Gated DeltaNet
// recurrence on Blackwell tensor cores (tcgen05 + TMEM, operands fed by TMA).
//
// Method: Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2":
//     S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t,
//     a_t = exp(g_t), g scalar per head or one value per key channel.
// The chunkwise mode ("Gated DeltaNet" entity trail, finding of 2026-07-29)
// computes the same mathematics with dense products inside a chunk.
//
// Chunk algebra (derived by unrolling the recurrence over a chunk of C = 64
// tokens with initial state S; G_r = cumulative sum of g inside the chunk,
// a scalar or a dk-vector; E_r = exp(G_r); u_r = b_r (v_r - S'_r^T k_r) is
// the corrected value the delta rule writes at token r):
//   A_rj = b_r k_r^T Diag(exp(G_r - G_j)) k_j          (j < r)
//   T    = (I + A)^{-1},  T' = T Diag(b)                (unit lower triangular)
//   W    = T' (K * E),    U = T' V - W S
//   P_rj = q_r^T Diag(exp(G_r - G_j)) k_j              (j <= r)
//   O    = (Q * E) S + P U
//   S   <- Diag(E_last) S + (K * D)^T U,  D_r = exp(G_last - G_r)
// The state S stays fp32 in registers across chunks.
//
// Per-channel decay inside A and P.  exp(G_r - G_j) per key channel is
// factored through a reference token m at the centre of a 32-token block:
// exp(G_r - G_m) * exp(G_m - G_j).  With g >= -5 (the gate domain of the
// model card, section 2.1, g = -min(softplus(.), 160/bs2), bs2 = 32) every
// factor lies within exp(+-80), inside fp32 and bf16 range, so A and P come
// out of plain matrix products (K * F)(K / F)^T.  Rows of block 0 (tokens
// 0-31) use reference 15, rows of block 1 use reference 47; both products
// share the left operand [K * F ; Q * F] and differ in the right one.
// The scalar gate needs no factorisation: exp(G_r - G_j) is applied exactly
// to K K^T and Q K^T after the product, for any g <= 0.
//
// Precision.  The output o is a small difference of much larger terms
// ((Q*E) S and P U; on the source's workloads max|o| ~ 9 rms(o)), so plain
// bf16 operands would cost more than a 2e-2 * rms(o) error budget.  The
// model card's kernel computes in "bf16x3" (section 3.2 Precision, section 5
// compute mode): a value is carried as a bf16 hi part plus a bf16 lo part
// and a product takes three bf16 MMAs (hi*hi + hi*lo + lo*hi).  Here that is
// applied to the operands that need it: the factored operands of A and P,
// T', P, U, Z and K*D.  The state copy S, K*E and Q*E, whose magnitudes stay
// moderate, are fp16 operands (4x finer than bf16).  Accumulation is fp32 in
// TMEM and the output is written in fp32.
//
// Products (all 128-row tcgen05.mma; transposed forms put the 128-wide key or
// value dimension on M):
//   X       = [K*F;Q*F] (K/F)^T       M = 2C rows, N = 64 / 96 -> A and P (raw)
//   [Y|O]^T = S^T [K*E; Q*E]^T        M = dv, N = 2C (Y^T = S^T (K*E)^T, O^T = S^T (Q*E)^T)
//   U^T     = Z^T T'^T, Z = V - Y      M = dv, N = C, K = C  (U = T' V - W S with W S = T' Y)
//   O^T    += U^T P^T                  M = dv, N = C
//   SN      = (K*D)^T U                M = dk, N = dv, K = C
//
// The phases of a chunk run one after another in one CTA per (batch, head,
// segment); with a scalar gate the state step of chunk c runs after chunk
// c + 1's gate scan and X issue (see finish_chunk), and the next chunk's TMA
// loads overlap the end of the chunk.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "chunk_common.cuh"
#include "warp_mma.cuh"
#include "gdn_internal.cuh"
#include "sm100_util.cuh"

namespace gdn {

__device__ unsigned int g_status_word = 0;

namespace {

using namespace sm100;
using namespace chunk;

constexpr int C = 64;      // chunk length
constexpr int D = 128;     // dk = dv
constexpr int NT = 256;    // threads per CTA

// ---- shared-memory map (byte offsets from a 1024-aligned base) -------------
// R_IN: raw K and Q of the chunk (TMA, bf16, 128B-swizzled rows):
//   [half][K rows 0-63 | Q rows 0-63][128 B].  Dead once the derived tiles
//   are built; then holds T' (hi, lo), the solve scratch and W^T.
constexpr uint32_t R_IN = 0;                 // 32 KB
constexpr uint32_t OFF_TH = R_IN;            //   8 KB T' hi [64 r][64 m]
constexpr uint32_t OFF_TL = R_IN + 8192;     //   8 KB T' lo
constexpr uint32_t OFF_Y = R_IN + 16384;     //   10 KB solve scratch 2 x [32][40] fp32
// (R_IN + 26 KB .. 32 KB unused)
constexpr uint32_t R_V = 32768;              // 16 KB raw V [half][64][128 B]
constexpr uint32_t R_S = 49152;              // 32 KB S fp16 [j half][128 i][64 j]
constexpr uint32_t R_X = 81920;              // 112 KB, two uses per chunk:
//  (a) X operands (per-channel gate), bf16 hi / lo:
constexpr uint32_t OFF_AH = R_X;             //   32 KB [half][K*F 64 | Q*F 64][128 B]
constexpr uint32_t OFF_AL = R_X + 32768;     //   32 KB
constexpr uint32_t OFF_CB = R_X + 65536;     //   48 KB [half][hi 96 rows | lo 96 rows][128 B]: rows 0-31
                                             //   K/F (ref 15), rows 32-95 K*exp(G_47 - G); one N = 96 B,
                                             //   and [hi; lo] one N = 192 B
constexpr uint32_t CB_HALF = 96 * 128;
//  (b) after X: derived tiles, P, solve input, U
constexpr uint32_t OFF_KE = R_X;             //   16 KB K*E fp16 [half][K*E 64 r | Q*E 64 r][128 B]:
constexpr uint32_t OFF_ZH = R_X;              //   after Y: Z^T = V^T - Y^T bf16 hi [128 j][64 r]
constexpr uint32_t OFF_OST = R_X;            //   at the chunk's end: 32 KB O fp32 [64 t][128 j] (TMA store)
constexpr uint32_t OFF_OST_LATE = R_X + 81920;  // scalar gate: the same, over A / T / U (see finish_chunk)
constexpr uint32_t OFF_QE = R_X + 8192;      //   16 KB Q*E fp16   one N = 128 B operand of Y and O
constexpr uint32_t OFF_ZL = R_X + 16384;      //   after Y and the first O products: Z^T lo
constexpr uint32_t OFF_KDH = R_X + 32768;    //   16 KB K*D bf16 hi
constexpr uint32_t OFF_KDL = R_X + 49152;    //   16 KB K*D bf16 lo
constexpr uint32_t OFF_PH = R_X + 65536;     //   8 KB P hi [64 r][64 m]
constexpr uint32_t OFF_PL = R_X + 73728;     //   8 KB P lo
constexpr uint32_t OFF_A = R_X + 81920;      //   16 KB A fp32 [64][64]
constexpr uint32_t OFF_TF = R_X + 98304;     //   16 KB T fp32 [64][64] (tidx layout)
constexpr uint32_t OFF_UH = R_X + 81920;     //   16 KB U^T hi [128 j][64 r] (after solve)
constexpr uint32_t OFF_UL = R_X + 98304;     //   16 KB U^T lo
constexpr uint32_t R_SMALL = R_X + 114688;
constexpr uint32_t SM_GAM = R_SMALL;          // 64 f32: scalar G
constexpr uint32_t SM_BETA = SM_GAM + 256;    // 64 f32
constexpr uint32_t SM_REF0 = SM_BETA + 256;   // 128 f32: G at token 15 (channel)
constexpr uint32_t SM_REF1 = SM_REF0 + 512;   // 128 f32: G at token 47
constexpr uint32_t SM_LAST = SM_REF1 + 512;   // 128 f32: G at token 63
constexpr uint32_t SM_ER = SM_LAST + 512;     // 64 f32: exp(G_r - G_31)  (scalar gate)
constexpr uint32_t SM_FJ = SM_ER + 256;       // 64 f32: exp(G_31 - G_j)
constexpr uint32_t SM_SAFE = SM_FJ + 256;     // int: product form in range
constexpr uint32_t SM_BAR = SM_SAFE + 16;     // 4 mbarriers: loads, products, products into O, SN
constexpr uint32_t SM_TMEM = SM_BAR + 32;     // TMEM base address
constexpr uint32_t SM_RED = SM_TMEM + 16;     // 8 f32: per-warp max |M| (transition CTAs)
constexpr uint32_t SMEM_USED = SM_RED + 32;

// A transition CTA stops once every entry of its M is at most this: from
// there on the dropped part of the correction is below 2^-53 |S_start|
// (see Params::trans_len).
constexpr float kTransitionDrop = 0x1p-60f;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

// ---- TMEM columns (512 allocated) -------------------------------------------
constexpr uint32_t TM_X = 0;      // X: 128 rows (A rows 0-63, P rows 64-127); scalar N = 64,
                                  //   per-channel N = 192 (hi / lo halves, summed on load)
constexpr uint32_t TM_YT = 192;   // Y^T = S^T (K*E)^T: 128 x 64
constexpr uint32_t TM_OT = 256;   // O^T: 128 x 64 (next to Y^T: one N = 128 product forms both)
constexpr uint32_t TM_UT = 320;   // U^T: 128 x 128, Z^T hi T'^T (hi + lo) side by side (summed on load)
constexpr uint32_t TM_SN = 384;   // SN:  128 x 128, over U^T's upper half (consumed before SN)

// One launch covers B x nseg x H (batch, time segment, head) problems, and
// optionally a second copy of them ("transition" CTAs, second half of the
// grid) that run the same chunk recursion with v = 0 from the identity state:
// the state map of a segment is affine, S_end = M S_start + S_end(0), and
// those CTAs produce M (dk x dk).
struct Params {
    const float* g;            // [B, T, H] or [B, T, H, D]
    const float* beta;         // [B, T, H]
    const float* state_in;     // [B, in_segs, H, D, D] or null (zero state)
    float* state_out;          // [B, out_segs, H, D, D] or null; out_segs == 1: last segment only
    float* trans_out;          // [B, nseg, H, D, D] transitions, or null (no transition CTAs)
    float* out;                // [B, T, H, D] fp32, or null (outputs not written)
    int T, H, B;
    int nseg, seg_len;         // time segments of seg_len tokens (a multiple of C)
    int in_segs, out_segs;     // 1 or nseg
    // Transition CTAs with a buffer here also form outputs: with v = 0 from
    // the identity their "output" is w_t = M_t^T q_t ([B, T, H, D] fp16),
    // M_t the state map from the segment start to token t, so that the true
    // output is the zero-start one plus S_start^T w_t.  (fp16: the
    // correction that reads w multiplies in fp16 anyway.)
    __half* wout = nullptr;
    // Segment 0 from the true initial state: its zero-start CTA reads
    // state_in (the others start from zero) and it has no transition CTA, so
    // that transition CTAs cover segments trans_first .. nseg - 1.
    int trans_first = 0;
    bool in_first_only = false;
    // Early end of the transitions ([B, nseg, H] chunks run; null: run every
    // chunk).  Every step of the recurrence is a contraction when g <= 0
    // (every channel of a per-channel gate), beta in [0, 1] and |k| = 1 (the
    // model card's input domain, section 2.1): |I - b k k^T|_2 <= 1 while
    // 0 <= b |k|^2 <= 2, and |Diag(exp(g))|_2 <= 1.  So once max |M_ij| <= kTransitionDrop after a chunk,
    // every later M_t' has |M_t'|_2 <= 128 kTransitionDrop = 2^-53, and
    // dropping it changes an output by at most 2^-53 |S_start|_2 |q| --
    // below fp32 resolution.  A transition CTA checks the domain on the
    // tokens it runs (g <= 0 and 0 <= b (K K^T)_rr <= 2, from the diagonal of
    // the product it forms anyway) and, before stopping, beta and g of the
    // tokens it would skip; it never stops once a token is outside.  It then
    // records how many chunks it ran (negated when it stopped early and
    // dropped M) and writes M = 0 and w only for those chunks; the correction
    // reads the count, and the combine skips a dropped M.  With decaying
    // gates M falls below the threshold within a chunk or two.
    int* trans_len = nullptr;
};

template <bool CHANNEL>
__global__ void __launch_bounds__(NT, 1)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const __grid_constant__ CUtensorMap tm_w, const Params p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (128B-swizzle atoms), derived by a pointer offset
    // so that the compiler keeps the shared address space (LDS/STS, not
    // generic loads and stores).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    float* sGam = reinterpret_cast<float*>(smem + SM_GAM);
    float* sBeta = reinterpret_cast<float*>(smem + SM_BETA);
    float* sRef0 = reinterpret_cast<float*>(smem + SM_REF0);
    float* sRef1 = reinterpret_cast<float*>(smem + SM_REF1);
    float* sLast = reinterpret_cast<float*>(smem + SM_LAST);
    float* sEr = reinterpret_cast<float*>(smem + SM_ER);
    float* sFj = reinterpret_cast<float*>(smem + SM_FJ);
    int* sSafe = reinterpret_cast<int*>(smem + SM_SAFE);
    float* sA = reinterpret_cast<float*>(smem + OFF_A);
    float* sTf = reinterpret_cast<float*>(smem + OFF_TF);
    float* sY = reinterpret_cast<float*>(smem + OFF_Y);
    const uint32_t bar_tma = sbase + SM_BAR;
    const uint32_t bar_mma = sbase + SM_BAR + 8;
    const uint32_t bar_out = sbase + SM_BAR + 16;   // O^T products, committed apart
    const uint32_t bar_sn = sbase + SM_BAR + 24;    // SN, committed apart
    uint32_t* sTmemBase = reinterpret_cast<uint32_t*>(smem + SM_TMEM);
    float* sRed = reinterpret_cast<float*>(smem + SM_RED);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int quad = warp & 3;      // TMEM lane quarter of this warp
    const int half = warp >> 2;     // which half of the columns this warp takes
    const int T = p.T;
    const int H = p.H;
    const int per_mode = p.B * p.nseg * H;
    const bool transition = static_cast<int>(blockIdx.x) >= per_mode;
    const int rem = static_cast<int>(blockIdx.x) - (transition ? per_mode : 0);
    const int nseg_here = transition ? p.nseg - p.trans_first : p.nseg;
    const int h = rem % H;
    const int seg = (transition ? p.trans_first : 0) + (rem / H) % nseg_here;
    const int b = rem / (H * nseg_here);
    const int t_begin = seg * p.seg_len;
    const int t_end = min(T, t_begin + p.seg_len);
    const int nchunks = t_end > t_begin ? (t_end - t_begin + C - 1) / C : 0;
    // Outputs are formed only where they are written (not by transition CTAs
    // nor by the zero-start pass of the segment path).
    const bool want_o = transition ? p.wout != nullptr : p.out != nullptr;
    const CUtensorMap* tm_store = transition ? &tm_w : &tm_o;

    // Element ownership for the gate prep and tile building: 16 channel
    // chunks of 8 (ck) x 16 lanes (tg), lane tg owning tokens tg + 16 u,
    // u = 0..3.  The 16 lanes of a channel chunk sit in one half-warp (the
    // cumulative sum is a shuffle scan) and eight consecutive lanes touch eight
    // consecutive rows of a 128B-swizzled tile (no shared-memory bank conflicts).
    const int ck = 2 * warp + (lane >> 4);
    const int tg = lane & 15;
    const int ckh = ck >> 3;       // 64-channel half of the tile
    const int ckc = ck & 7;        // 16-byte chunk within a 128-byte row

    if (tid == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (want_o) prefetch_tensormap(tm_store);
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_out, 1);
        mbar_init(bar_sn, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + SM_TMEM, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmemBase;

    // ---- resident fp32 state: thread owns row i, columns [64*half, +64) ------
    const int srow = quad * 32 + lane;
    const int scol = half * 64;
    float s[64];
    const long DD = (long)D * D;
    if (transition) {                       // identity: the chain yields M
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = (srow == scol + c) ? 1.f : 0.f;
    } else if (p.state_in && (!p.in_first_only || seg == 0)) {
        const long sin_b = (((long)b * p.in_segs + (p.in_segs == 1 ? 0 : seg)) * H + h) * DD;
        const float4* src = reinterpret_cast<const float4*>(p.state_in + sin_b + (long)srow * D + scol);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float4 t = src[c];
            s[4 * c] = t.x; s[4 * c + 1] = t.y; s[4 * c + 2] = t.z; s[4 * c + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = 0.f;
    }
    // fp16 copy: MN-major tile [j half][128 i rows][64 j] (row i, 8 chunks).
    auto write_state_f16 = [&]() {
        uint8_t* dst = smem + R_S + half * 16384;
#pragma unroll
        for (int c = 0; c < 8; ++c) store_f16x8(dst + swz(srow, c), &s[8 * c]);
    };
    write_state_f16();

    auto issue_loads = [&](int chunk) {
        const int t0 = t_begin + chunk * C;
        mbar_expect_tx(bar_tma, (transition ? 2 : 3) * 16384);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sbase + R_IN + hf * 16384, &tm_k, hf * 64, h, t0, b, bar_tma);
            tma_load_4d(sbase + R_IN + hf * 16384 + 8192, &tm_q, hf * 64, h, t0, b, bar_tma);
            if (!transition) tma_load_4d(sbase + R_V + hf * 8192, &tm_v, hf * 64, h, t0, b, bar_tma);
        }
    };

    fence_async_smem();
    __syncthreads();
    if (tid == 0 && nchunks > 0) issue_loads(0);
    int tma_waited = -1;   // last chunk whose loads were waited for
    int tma_issued = nchunks > 0 ? 1 : 0;   // chunks whose loads were issued (tid 0)
    // Transition CTAs that may stop early: this thread has seen a token
    // outside the contracting domain (sticky), and the chunks run so far.
    const bool may_stop = transition && p.trans_len != nullptr;
    bool outside = false;
    bool stopped = false;
    int chunks_run = nchunks;

    uint32_t mma_phase = 0;
    bool ok = true;
    auto mma_sync = [&]() {   // all threads wait for the last commit
        ok = ok && mbar_wait(bar_mma, mma_phase, &g_status_word);
        mma_phase ^= 1;
        tc_fence_after();
    };

    // g (per-channel: this thread's 4 tokens x 8 channels) and, in warp 0,
    // beta and the scalar g are loaded into registers one chunk ahead, issued
    // after a shared-memory proxy fence (which would wait for them).
    auto load_gate = [&](int chunk, float (&gn)[4][8]) {
        const int tc0 = t_begin + chunk * C;
        const long tkc = ((long)b * T + tc0) * H + h;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = tg + 16 * u;
            if (tc0 + r < t_end) {
                const float4* src = reinterpret_cast<const float4*>(p.g + (tkc + (long)r * H) * D + 8 * ck);
                const float4 a = src[0], c = src[1];
                gn[u][0] = a.x; gn[u][1] = a.y; gn[u][2] = a.z; gn[u][3] = a.w;
                gn[u][4] = c.x; gn[u][5] = c.y; gn[u][6] = c.z; gn[u][7] = c.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gn[u][e] = 0.f;
            }
        }
    };
    auto load_beta = [&](int chunk, float (&bg)[4]) {   // warp 0: lane, 32 + lane
        bg[0] = bg[1] = bg[2] = bg[3] = 0.f;
        if (warp != 0) return;
        const int tc0 = t_begin + chunk * C;
        const long tkc = ((long)b * T + tc0) * H + h;
        if (tc0 + lane < t_end) {
            bg[0] = p.beta[tkc + (long)lane * H];
            if (!CHANNEL) bg[2] = p.g[tkc + (long)lane * H];
        }
        if (tc0 + 32 + lane < t_end) {
            bg[1] = p.beta[tkc + (long)(32 + lane) * H];
            if (!CHANNEL) bg[3] = p.g[tkc + (long)(32 + lane) * H];
        }
    };
    float gnext[4][8], bgnext[4];
    if (CHANNEL && nchunks > 0) load_gate(0, gnext);
    if (nchunks > 0) load_beta(0, bgnext);

    // With a scalar gate the next chunk's X product reads only the raw K and Q
    // (R_IN), so the state step of chunk c can follow the issue of chunk
    // c + 1's X (see finish_chunk).
    constexpr bool LATE = !CHANNEL;
    constexpr uint32_t OST = LATE ? OFF_OST_LATE : OFF_OST;
    float e_last = 1.f;       // E_last of the chunk whose state step is due
    uint32_t sn_phase = 0;
    int pending = -1;         // LATE: the chunk whose state step is due
    // The state update and output of chunk cj: S <- Diag(E_last) S + SN, its
    // fp16 copy for the next chunk's products, O (or w) to shared memory and
    // one TMA store, and a transition's early end.  0: go on, 1: abandoned
    // (a bounded wait ran out), 2: the transition ended early.  With a scalar
    // gate (LATE) it runs one chunk late, after the next chunk's gate prep and
    // the issue of its X product, so that those overlap the SN and O products;
    // its O goes to a staging tile clear of the next chunk's derived tiles.
    auto finish_chunk = [&](int cj) -> int {
        const int tj0 = t_begin + cj * C;
        ok = ok && mbar_wait(bar_sn, sn_phase, &g_status_word);
        sn_phase ^= 1;
        tc_fence_after();
        float o[32];
        {
            const uint32_t lb = tmem + (static_cast<uint32_t>(quad * 32) << 16);
            {
                float sn0[32], sn1[32];
                tmem_ld32(lb + TM_SN + half * 64, sn0);
                tmem_ld32(lb + TM_SN + half * 64 + 32, sn1);
                tmem_wait_ld();
                const float2 e2 = make_float2(e_last, e_last);
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 a = fma2(e2, make_float2(s[c], s[c + 1]), make_float2(sn0[c], sn0[c + 1]));
                    const float2 z = fma2(e2, make_float2(s[32 + c], s[33 + c]), make_float2(sn1[c], sn1[c + 1]));
                    s[c] = a.x; s[c + 1] = a.y; s[32 + c] = z.x; s[33 + c] = z.y;
                }
            }
            write_state_f16();
            if (want_o) {
                ok = ok && mbar_wait(bar_out, cj & 1, &g_status_word);
                tc_fence_after();
                tmem_ld32(lb + TM_OT + half * 32, o);
                tmem_wait_ld();
                // O^T (lane = value column) -> [token][column] fp32 over the
                // consumed K*E / Q*E tiles; one TMA store per chunk, rows past
                // T dropped.  Thread stores would hold up the next proxy fence.
                if (transition) {   // w in fp16
                    __half* sh = reinterpret_cast<__half*>(smem + OST) + half * 32 * D + srow;
#pragma unroll
                    for (int r = 0; r < 32; ++r) sh[r * D] = __float2half_rn(o[r]);
                } else {
                    float* so = reinterpret_cast<float*>(smem + OST) + half * 32 * D + srow;
#pragma unroll
                    for (int r = 0; r < 32; ++r) so[r * D] = o[r];
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (may_stop) {   // this chunk's max |M| (or +inf outside the domain), per warp
            float m = 0.f;
#pragma unroll
            for (int c = 0; c < 64; ++c) m = fmaxf(m, fabsf(s[c]));
            if (outside) m = __int_as_float(0x7f800000);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) sRed[warp] = m;
        }
        if (__syncthreads_or(!ok)) return 1;
        if (want_o && tid == 0) {
            tma_store_4d(tm_store, sbase + OST, 0, h, tj0, b);
            bulk_commit();
        }
        if (may_stop && cj + 1 < nchunks) {
            // Read by every thread between this barrier and the next chunk's
            // first one; rewritten only at the next chunk's end.
            float m = sRed[0];
#pragma unroll
            for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, sRed[w]);
            if (m <= kTransitionDrop) {
                // The tokens not run must be inside the domain too: scan their
                // beta and g (8 bytes a token; 4 + 4 dk with a per-channel
                // gate); unit keys are the caller's contract.
                bool bad = false;
                if (!CHANNEL) {
                    for (long t = tj0 + C + tid; t < t_end; t += NT) {
                        const long i = ((long)b * T + t) * H + h;
                        const float bt = p.beta[i], gt = p.g[i];
                        bad |= !(bt >= 0.f && bt <= 1.f && gt <= 0.f);
                    }
                } else {
                    const long nt = t_end - (tj0 + C);
                    for (long e = tid; e < nt * (D / 4); e += NT) {
                        const long i = ((long)b * T + tj0 + C + e / (D / 4)) * H + h;
                        const float4 gv = reinterpret_cast<const float4*>(p.g + i * D)[e % (D / 4)];
                        bad |= !(gv.x <= 0.f && gv.y <= 0.f && gv.z <= 0.f && gv.w <= 0.f);
                        if (e % (D / 4) == 0) bad |= !(p.beta[i] >= 0.f && p.beta[i] <= 1.f);
                    }
                }
                if (!__syncthreads_or(bad)) {
                    stopped = true;
                    chunks_run = cj + 1;
                    return 2;
                }
                outside = true;   // some later token is outside: run every chunk
            }
        }
        return 0;
    };

    for (int ci = 0; ci < nchunks; ++ci) {
        const int t0 = t_begin + ci * C;
        const long tk0 = ((long)b * T + t0) * H + h;     // flat (b, t0, h)

        // ---------------------------------------------------- gate prep --------
        // Per-channel: this thread's 4 tokens x 8 channels of g, cumulated over
        // the chunk (registers).  Scalar: warp 0 scans the 64 values.
        float gam[4][8];
        if (CHANNEL) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int e = 0; e < 8; ++e) gam[u][e] = gnext[u][e];
            if (may_stop) {   // this thread's 4 tokens x 8 channels of g (0 past T)
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (!(gnext[u][e] <= 0.f)) outside = true;
            }
            // Inclusive scan over the 16 lanes of each 16-token block, then add
            // the totals of the preceding blocks.
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float x = __shfl_up_sync(0xffffffffu, gam[u][e], o, 16);
                        if (tg >= o) gam[u][e] += x;
                    }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float off = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float tot = __shfl_sync(0xffffffffu, gam[u][e], 15, 16);
                    gam[u][e] += off;
                    off += tot;
                }
            }
            if (ci + 2 < nchunks) {   // warm L2 two chunks ahead
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = 2 * C + tg + 16 * u;
                    if (t0 + r < t_end) prefetch_l2(p.g + (tk0 + (long)r * H) * D + 8 * ck);
                }
            }
            if (tg == 15) {   // G at tokens 15, 47 (block references) and 63
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sRef0[8 * ck + e] = gam[0][e];
                    sRef1[8 * ck + e] = gam[2][e];
                    sLast[8 * ck + e] = gam[3][e];
                }
            }
        }
        if (warp == 0) {
            const float b0 = bgnext[0], b1 = bgnext[1];
            float g0 = bgnext[2], g1 = bgnext[3];
            sBeta[lane] = b0;
            sBeta[32 + lane] = b1;
            if (!CHANNEL && may_stop && !(g0 <= 0.f && g1 <= 0.f)) outside = true;
            if (!CHANNEL) {
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float x0 = __shfl_up_sync(0xffffffffu, g0, o);
                    const float x1 = __shfl_up_sync(0xffffffffu, g1, o);
                    if (lane >= o) { g0 += x0; g1 += x1; }
                }
                g1 += __shfl_sync(0xffffffffu, g0, 31);
                sGam[lane] = g0;
                sGam[32 + lane] = g1;
                // exp(G_r - G_j) = exp(G_r - G_31) exp(G_31 - G_j), exact in fp32
                // while the chunk's total decay is at most 80; otherwise the
                // epilogue exponentiates directly.
                const float m = __shfl_sync(0xffffffffu, g0, 31);
                float mx = fmaxf(g0, g1), mn = fminf(g0, g1);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                }
                sEr[lane] = __expf(g0 - m);
                sEr[32 + lane] = __expf(g1 - m);
                sFj[lane] = __expf(m - g0);
                sFj[32 + lane] = __expf(m - g1);
                if (lane == 0) *sSafe = (mx - mn) <= 80.f;
            }
        }
        ok = ok && mbar_wait(bar_tma, ci & 1, &g_status_word);
        if (ok) tma_waited = ci;    // else the exit path drains these loads
        if (tid == 0) bulk_wait_read_all();   // the previous output store has read OFF_OST
        if (__syncthreads_or(!ok)) break;

        // ---------------------------------------------------- X = raw A and P --
        if (CHANNEL) {
            // Factored operands, bf16 hi + lo (see header).
            // Channel pairs on the paired fp32 instructions; tokens tg + 16u
            // with u < 2 are before token 32 (reference 15).
            const float2 l2e = make_float2(kLog2e, kLog2e);
            float2 ref0[4], ref1[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ref0[e] = make_float2(sRef0[8 * ck + 2 * e], sRef0[8 * ck + 2 * e + 1]);
                ref1[e] = make_float2(sRef1[8 * ck + 2 * e], sRef1[8 * ck + 2 * e + 1]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = tg + 16 * u;
                float kf[8], qf[8];
                load_bf16x8(smem + R_IN + ckh * 16384 + swz(r, ckc), kf);
                load_bf16x8(smem + R_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
                float2 kr[4], qr[4], kc[4], kc1[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 k2 = make_float2(kf[2 * e], kf[2 * e + 1]);
                    const float2 q2 = make_float2(qf[2 * e], qf[2 * e + 1]);
                    const float2 g2 = make_float2(gam[u][2 * e], gam[u][2 * e + 1]);
                    const float2 xl = mul2(sub2(g2, u < 2 ? ref0[e] : ref1[e]), l2e);
                    const float2 F = make_float2(ex2_approx(xl.x), ex2_approx(xl.y));
                    const float2 Fi = make_float2(ex2_approx(-xl.x), ex2_approx(-xl.y));
                    kr[e] = mul2(k2, F);
                    qr[e] = mul2(q2, F);
                    kc[e] = mul2(k2, Fi);
                    if (u < 2) {
                        const float2 yl = mul2(sub2(ref1[e], g2), l2e);
                        kc1[e] = mul2(k2, make_float2(ex2_approx(yl.x), ex2_approx(yl.y)));
                    } else {
                        kc1[e] = kc[e];
                    }
                }
                const uint32_t o128 = ckh * 16384 + swz(r, ckc);
                const uint32_t o128q = ckh * 16384 + swz(64 + r, ckc);
                store_split2(smem + OFF_AH + o128, smem + OFF_AL + o128, kr);
                store_split2(smem + OFF_AH + o128q, smem + OFF_AL + o128q, qr);
                if (u < 2) {
                    const uint32_t o32 = ckh * 2 * CB_HALF + swz(r, ckc);
                    store_split2(smem + OFF_CB + o32, smem + OFF_CB + CB_HALF + o32, kc);
                }
                const uint32_t o64 = ckh * 2 * CB_HALF + swz(32 + r, ckc);
                store_split2(smem + OFF_CB + o64, smem + OFF_CB + CB_HALF + o64, kc1);
            }
            fence_async_smem();
            __syncthreads();
            if (ci + 1 < nchunks) load_gate(ci + 1, gnext);
        }
        if (tid == 0) {
            tc_fence_after();
            if (CHANNEL) {
                // A hi times [B hi; B lo] (N = 192), A lo times B hi into the
                // first 96 columns; the A/P epilogue adds the halves.
                const uint32_t id2 = idesc_bf16(128, 192, false, false);
                const uint32_t id = idesc_bf16(128, 96, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ka = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t kb = (ks >> 2) * 2 * CB_HALF + (ks & 3) * 32;
                    const uint64_t ah = sdesc_sw128(sbase + OFF_AH + ka, 16, 1024);
                    const uint64_t al = sdesc_sw128(sbase + OFF_AL + ka, 16, 1024);
                    const uint64_t bh = sdesc_sw128(sbase + OFF_CB + kb, 16, 1024);
                    mma_bf16(tmem + TM_X, ah, bh, id2, ks > 0);
                    mma_bf16(tmem + TM_X, al, bh, id, 1);
                }
            } else {
                // Exact: bf16 inputs, fp32 accumulation.
                const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = sdesc_sw128(sbase + R_IN + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    mma_bf16(tmem + TM_X, a, a, id, ks > 0);
                }
            }
            mma_commit(bar_mma);
        }
        // Per-channel X reads its operands from R_X, where the derived tiles
        // go: wait first.  With a scalar gate X reads only the raw K and Q, so
        // the derived tiles are built while it runs.
        if (CHANNEL) {
            mma_sync();
            if (__syncthreads_or(!ok)) break;
        }
        if (LATE && ci > 0) {
            const int r = finish_chunk(ci - 1);
            pending = -1;
            if (r != 0) {
                if (r == 2) mma_sync();      // ended early: this chunk's X is in flight
                break;
            }
        }
        if (ci + 1 < nchunks) load_beta(ci + 1, bgnext);

        // ------------------------------- derived tiles; A and P from X ----------
        // K*E (bf16), Q*E (fp16), K*D (bf16 hi + lo) into the freed X region.
        {
            const float2 l2e = make_float2(kLog2e, kLog2e);
            float2 last2[4];
            if (CHANNEL) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    last2[e] = make_float2(sLast[8 * ck + 2 * e], sLast[8 * ck + 2 * e + 1]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = tg + 16 * u;
                float kf[8], qf[8], ke[8], qe[8];
                float2 kd[4];
                load_bf16x8(smem + R_IN + ckh * 16384 + swz(r, ckc), kf);
                load_bf16x8(smem + R_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
                float2 E2 = make_float2(0.f, 0.f), D2 = E2;
                if (!CHANNEL) {
                    const float E = ex2_approx(sGam[r] * kLog2e);
                    const float Dd = ex2_approx((sGam[C - 1] - sGam[r]) * kLog2e);
                    E2 = make_float2(E, E);
                    D2 = make_float2(Dd, Dd);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 k2 = make_float2(kf[2 * e], kf[2 * e + 1]);
                    const float2 q2 = make_float2(qf[2 * e], qf[2 * e + 1]);
                    if (CHANNEL) {
                        const float2 g2 = make_float2(gam[u][2 * e], gam[u][2 * e + 1]);
                        const float2 el = mul2(g2, l2e);
                        const float2 dl = mul2(sub2(last2[e], g2), l2e);
                        E2 = make_float2(ex2_approx(el.x), ex2_approx(el.y));
                        D2 = make_float2(ex2_approx(dl.x), ex2_approx(dl.y));
                    }
                    const float2 ke2 = mul2(k2, E2), qe2 = mul2(q2, E2);
                    ke[2 * e] = ke2.x; ke[2 * e + 1] = ke2.y;
                    qe[2 * e] = qe2.x; qe[2 * e + 1] = qe2.y;
                    kd[e] = mul2(k2, D2);
                }
                const uint32_t o64 = ckh * 8192 + swz(r, ckc);
                const uint32_t o128 = ckh * 16384 + swz(r, ckc);
                store_f16x8(smem + OFF_KE + o128, ke);
                store_f16x8(smem + OFF_QE + o128, qe);
                store_split2(smem + OFF_KDH + o64, smem + OFF_KDL + o64, kd);
            }
        }
        fence_async_smem();                  // K*E, Q*E -> the products below
        if (!CHANNEL) mma_sync();            // X
        // LATE: the previous chunk's output store has read its staging tile,
        // which the A/P epilogue below overwrites.
        if (LATE && tid == 0) bulk_wait_read_all();
        if (__syncthreads_or(!ok)) break;
        // Y^T = S^T (K*E)^T and O^T = S^T (Q*E)^T: the state-dependent
        // products that need only this chunk's derived tiles, issued now, so
        // that they run during the A/P epilogue.  The corrected values follow
        // as U = T' (V - (K*E) S) = T' Z (W S = T' (K*E) S), one product after
        // the solve instead of W^T and U~^T, then U^T -= S^T W^T.
        // With outputs, one N = 128 product over [K*E; Q*E] forms Y^T (TMEM
        // columns TM_YT ..) and O^T (TM_OT = TM_YT + 64 ..) together.
        static_assert(TM_OT == TM_YT + 64, "Y^T and O^T side by side");
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_y = idesc_f16(128, want_o ? 128 : 64, true, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + R_S + ks * 2048, 16384, 1024);
                const uint64_t bk = sdesc_sw128(sbase + OFF_KE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                mma_bf16(tmem + TM_YT, a, bk, id_y, ks > 0);
            }
            mma_commit(bar_mma);
        }
        // P (rows 64-127, warps of lane quadrants 2 and 3) only where outputs
        // are formed.
        if (quad < 2 || want_o) {
            // Thread: row L = TMEM lane of X (A rows 0-63, P rows 64-127),
            // columns j in [32*half, 32*half + 32).
            const int L = quad * 32 + lane;
            const bool is_p = L >= 64;
            const int r = L & 63;
            float x[32];
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
            bool zero = false;
            if (CHANNEL) {
                // block 0: X columns 0-31 hold j = 0..31; block 1: columns
                // 32-95 hold j = 0..63; the lo half 96 columns further on.
                // (The lo half in two 16-column loads keeps the registers
                // the per-channel kernel has.)
                const uint32_t col = r < 32 ? 0u : 32u + half * 32u;
                zero = r < 32 && half != 0;
                if (!zero) {
                    float x2[16];
                    tmem_ld32(lane_base + TM_X + col, x);
                    tmem_ld16(lane_base + TM_X + 96 + col, x2);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) x[jj] += x2[jj];
                    tmem_ld16(lane_base + TM_X + 96 + col + 16, x2);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) x[16 + jj] += x2[jj];
                }
            } else {
                tmem_ld32(lane_base + TM_X + half * 32, x);
                tmem_wait_ld();
            }
            if (zero) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) x[jj] = 0.f;
            }
            const float br = sBeta[r];
            const float Gr = CHANNEL ? 0.f : sGam[r];
            const bool prod = !CHANNEL && *sSafe;
            const float er = CHANNEL ? 1.f : sEr[r];
            auto decay = [&](int j) -> float {
                if (CHANNEL) return 1.f;
                return prod ? er * sFj[j] : __expf(Gr - sGam[j]);
            };
            const int j0 = half * 32;
            if (!is_p) {
                if (may_stop && half == (r >> 5)) {   // this thread holds (K K^T)_rr = |k_r|^2
                    float xd = 0.f;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) xd = jj == (r & 31) ? x[jj] : xd;
                    if (!(br >= 0.f && br * xd <= 2.f)) outside = true;
                }
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    float a[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = j0 + 4 * j4 + e;
                        float val = 0.f;
                        if (j < r) val = br * x[4 * j4 + e] * decay(j);
                        a[e] = val;
                    }
                    *reinterpret_cast<float4*>(&sA[fidx(r, j0 + 4 * j4)]) = make_float4(a[0], a[1], a[2], a[3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float pv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = j0 + 8 * c + e;
                        float val = 0.f;
                        if (j <= r) val = x[8 * c + e] * decay(j);
                        pv[e] = val;
                    }
                    const int cc = half * 4 + c;
                    store_split(smem + OFF_PH + swz(r, cc), smem + OFF_PL + swz(r, cc), pv);
                }
            }
        }
        // Decay of the state over the whole chunk, per key row (own row).
        e_last = __expf(CHANNEL ? sLast[srow] : sGam[C - 1]);

        // Z^T = V^T - Y^T -> bf16 hi + lo [128 j][64 r] over the consumed K*E
        // and Q*E tiles (thread: value column j = srow, 32 tokens).
        mma_sync();                          // Y (and the first O products)
        {
            float z[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_YT + half * 32, z);
            tmem_wait_ld();
            if (!transition) {               // transition CTAs have V = 0
                const uint8_t* vcol = smem + R_V + (srow >> 6) * 8192 + ((srow & 7) << 1);
                const uint32_t vchunk = (srow & 63) >> 3;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = half * 32 + i;
                    const float vr = __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16*>(vcol + swz(r, vchunk)));
                    z[i] = vr - z[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = -z[i];
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
                store_split(smem + OFF_ZH + swz(srow, half * 4 + c), smem + OFF_ZL + swz(srow, half * 4 + c),
                            &z[8 * c]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---------------------------------------------------- T = (I + A)^{-1} --
        solve_unit_lower64_rd(sA, sTf, sY, tid);
        // T' = T Diag(beta) -> bf16 hi + lo, K-major [64 r][64 m].
        for (int e = tid; e < 512; e += NT) {
            const int r = e >> 3, c = e & 7;
            const float4 t0v = *reinterpret_cast<const float4*>(&sTf[tidx(r, 8 * c)]);
            const float4 t1v = *reinterpret_cast<const float4*>(&sTf[tidx(r, 8 * c + 4)]);
            const float tt[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
            float tv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int m = 8 * c + q;
                tv[q] = (m <= r) ? tt[q] * sBeta[m] : 0.f;
            }
            store_split(smem + OFF_TH + swz(r, c), smem + OFF_TL + swz(r, c), tv);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---------------------------------------------------- U^T = Z^T T'^T ---
        // bf16 hi + lo on both sides, three products per k-step.
        if (tid == 0) {
            tc_fence_after();
            // Z^T hi times [T' hi; T' lo] (one N = 128 operand: T' lo follows
            // T' hi) into columns TM_UT .. + 127, Z^T lo times T' hi into the
            // first 64; the epilogue adds the two halves.
            static_assert(OFF_TL == OFF_TH + 8192, "T' hi and lo as one operand");
            const uint32_t id2 = idesc_bf16(128, 128, false, false);
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t zh = sdesc_sw128(sbase + OFF_ZH + ks * 32, 16, 1024);
                const uint64_t zl = sdesc_sw128(sbase + OFF_ZL + ks * 32, 16, 1024);
                const uint64_t th = sdesc_sw128(sbase + OFF_TH + ks * 32, 16, 1024);
                mma_bf16(tmem + TM_UT, zh, th, id2, ks > 0);
                mma_bf16(tmem + TM_UT, zl, th, id, 1);
            }
            mma_commit(bar_mma);
        }
        mma_sync();
        if (__syncthreads_or(!ok)) break;
        // Raw K, Q, V, T' and Z are no longer read: prefetch the next chunk.
        if (tid == 0 && ci + 1 < nchunks) {
            issue_loads(ci + 1);
            ++tma_issued;
        }

        // U^T -> bf16 hi + lo [128 j][64 r] (K-major B of SN, K-major A of O^T).
        {
            float u[32], u2[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_UT + half * 32, u);
            tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_UT + 64 + half * 32, u2);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] += u2[i];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                store_split(smem + OFF_UH + swz(srow, half * 4 + c), smem + OFF_UL + swz(srow, half * 4 + c),
                            &u[8 * c]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ------------------------------- SN = (K D)^T U ; O^T += U^T P^T --------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_s = idesc_bf16(128, 128, true, false);
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t kdh = sdesc_sw128(sbase + OFF_KDH + ks * 2048, 8192, 1024);
                const uint64_t kdl = sdesc_sw128(sbase + OFF_KDL + ks * 2048, 8192, 1024);
                const uint64_t uh = sdesc_sw128(sbase + OFF_UH + ks * 32, 16, 1024);
                const uint64_t ul = sdesc_sw128(sbase + OFF_UL + ks * 32, 16, 1024);
                mma_bf16(tmem + TM_SN, kdh, uh, id_s, ks > 0);
                mma_bf16(tmem + TM_SN, kdh, ul, id_s, 1);
                mma_bf16(tmem + TM_SN, kdl, uh, id_s, 1);
            }
            mma_commit(bar_sn);
            if (want_o) {
                // (U^T hi times [P hi; P lo] as one N = 128 product, summed on
                // load, measured 0.5 % slower with a scalar gate.)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t uh = sdesc_sw128(sbase + OFF_UH + ks * 32, 16, 1024);
                    const uint64_t ul = sdesc_sw128(sbase + OFF_UL + ks * 32, 16, 1024);
                    const uint64_t ph = sdesc_sw128(sbase + OFF_PH + ks * 32, 16, 1024);
                    const uint64_t pl = sdesc_sw128(sbase + OFF_PL + ks * 32, 16, 1024);
                    mma_bf16(tmem + TM_OT, uh, ph, id_o, 1);
                    mma_bf16(tmem + TM_OT, uh, pl, id_o, 1);
                    mma_bf16(tmem + TM_OT, ul, ph, id_o, 1);
                }
                mma_commit(bar_out);
            }
        }
        if (LATE) {
            pending = ci;                // its state and output: next iteration
        } else {
            const int r = finish_chunk(ci);
            if (r != 0) break;
        }
    }
    if (LATE && pending >= 0 && ok) finish_chunk(pending);
    if (tid == 0) bulk_wait_all();     // output stores complete before exit
    if (tid == 0 && stopped && tma_issued > tma_waited + 1)   // the next chunk's loads
        mbar_wait(bar_tma, (tma_waited + 1) & 1, &g_status_word);
    if (tid == 0 && may_stop && ok)   // negative: stopped early, M dropped
        p.trans_len[((long)b * p.nseg + seg) * H + h] = stopped ? -chunks_run : chunks_run;

    if (!ok && tid == 0) {
        // Abandoned: drain what this CTA still has in flight (bounded) before
        // its shared memory and TMEM go away.
        if (tma_issued > tma_waited + 1) mbar_wait(bar_tma, (tma_waited + 1) & 1, &g_status_word);
        mma_commit(bar_mma);
        mbar_wait(bar_mma, mma_phase, &g_status_word);
    }
    float* sdst = nullptr;
    if (transition) {
        sdst = p.trans_out + (((long)b * p.nseg + seg) * H + h) * DD;
        if (stopped) {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = 0.f;   // the dropped transition
        }
    } else if (p.state_out != nullptr && (p.out_segs != 1 || seg == p.nseg - 1)) {
        sdst = p.state_out + (((long)b * p.out_segs + (p.out_segs == 1 ? 0 : seg)) * H + h) * DD;
    }
    if (ok && sdst) {
        float4* dst = reinterpret_cast<float4*>(sdst + (long)srow * D + scol);
#pragma unroll
        for (int c = 0; c < 16; ++c) dst[c] = make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- host side ---------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // The driver entry point is the same for every device; a function-local
    // static is initialised once, thread-safely.
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return nullptr;
    }();
    return fn;
}

// 4-D map over a bf16 [B, T, H, 128] tensor; box {64 channels, 1, 64 tokens, 1},
// 128-byte swizzle (the operand layout of the MMAs).
// out [B, T, H, 128] fp32, box = one chunk of one head, no swizzle.
bool make_out_map(CUtensorMap* map, const void* base, int H, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4, (cuuint64_t)T * H * D * 4};
    cuuint32_t box[4] = {(cuuint32_t)D, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// w [B, T, H, D] fp16, box = one chunk of one head, no swizzle.
bool make_half_map(CUtensorMap* map, const void* base, int H, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)D, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* map, const void* base, int H, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Serial combine of the segments' affine state maps, for one (batch, head)
// and a 32-column slice of the state:
//     S_start(0) = S0,   S_start(s + 1) = M_s S_start(s) + S_end(0)(s).
// In place: on entry seg_states[s] holds S_end(0)(s), the end state of
// segment s started from zero; on exit it holds S_start(s).  With seg0_true,
// seg_states[0] already holds the true end state of segment 0 (it ran from
// S0), so S_start(1) = seg_states[0] and M_0 is not read.  The state after
// the last segment goes to state_out (may alias state_in).  fp32 throughout.
constexpr int CB_COLS = 32;
__global__ void __launch_bounds__(256)
combine_segments_kernel(float* seg_states, const float* trans, const float* state_in,
                        float* state_out, int H, int nseg, int seg0_true, const int* trans_len)
{
    __shared__ __align__(16) float sS[D][CB_COLS];     // current state slice
    const int nslice = D / CB_COLS;
    const int slice = blockIdx.x % nslice;
    const int bh = blockIdx.x / nslice;                // b * H + h
    const int b = bh / H, h = bh % H;
    const int c0 = slice * CB_COLS;
    const int tid = threadIdx.x;
    const int i = tid >> 1, jc = (tid & 1) * 16;       // row i, 16 columns
    const long DD = (long)D * D;
    for (int e = tid; e < D * CB_COLS; e += 256) {
        const int r = e / CB_COLS, c = e % CB_COLS;
        sS[r][c] = state_in ? state_in[(long)bh * DD + (long)r * D + c0 + c] : 0.f;
    }
    __syncthreads();
    for (int sg = 0; sg < nseg; ++sg) {
        const long base = (((long)b * nseg + sg) * H + h) * DD;
        float* slot = seg_states + base + (long)i * D + c0 + jc;
        float acc[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = reinterpret_cast<const float4*>(slot)[q];
            acc[4 * q] = v.x; acc[4 * q + 1] = v.y; acc[4 * q + 2] = v.z; acc[4 * q + 3] = v.w;
        }
        const float4* mrow = reinterpret_cast<const float4*>(trans + base + (long)i * D);
        // No product where M is zero: segment 0 run from the true start, or a
        // transition that ended early (negative count, see Params::trans_len).
        const bool no_m = (sg == 0 && seg0_true) ||
                          (trans_len && sg >= 1 && trans_len[((long)b * nseg + sg) * H + h] < 0);
#pragma unroll 4
        for (int k4 = 0; k4 < (no_m ? 0 : D / 4); ++k4) {
            const float4 m = mrow[k4];
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float* srow_k = &sS[4 * k4 + e][jc];
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] = fmaf(mk[e], srow_k[c], acc[c]);
            }
        }
        float cur[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) cur[c] = sS[i][jc + c];
        __syncthreads();                               // every read of sS is done
#pragma unroll
        for (int q = 0; q < 4; ++q)
            reinterpret_cast<float4*>(slot)[q] =
                make_float4(cur[4 * q], cur[4 * q + 1], cur[4 * q + 2], cur[4 * q + 3]);
#pragma unroll
        for (int c = 0; c < 16; ++c) sS[i][jc + c] = acc[c];
        __syncthreads();
    }
    if (state_out) {
        for (int e = tid; e < D * CB_COLS; e += 256) {
            const int r = e / CB_COLS, c = e % CB_COLS;
            state_out[(long)bh * DD + (long)r * D + c0 + c] = sS[r][c];
        }
    }
}

// Segment correction: out[b, t, h, :] += S_start(b, seg(t), h)^T w[b, t, h, :]
// for every token of a segment, after the combine has produced the true start
// states.  One CTA per group of CORR_TILES 64-token tiles of one (batch,
// segment, head).  The term is a correction of the zero-start output: its
// products run single-pass in fp16 (about 2^-11 relative, inside the
// prefill's error budget), the start state as one fp16 tile read with
// ldmatrix, and the tiles of w (tokens x key channels) arrive through two
// cp.async stages while the previous tile's products run.
constexpr int CORR_TILES = 16;
struct __align__(16) CorrSmem {
    __half s[D][D + 8];
    __half w[2][C][D + 8];
};
__device__ __forceinline__ void corr_cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src) : "memory");
}
__global__ void __launch_bounds__(256, 2)
segment_correction_kernel(const float* __restrict__ seg_states, const __half* __restrict__ wbuf,
                          float* __restrict__ out, int T, int H, int nseg, int seg_len, int seg_first,
                          const int* __restrict__ trans_len)
{
    using namespace wmma16;
    extern __shared__ __align__(16) unsigned char corr_raw[];
    CorrSmem& m = *reinterpret_cast<CorrSmem*>(corr_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y % H, seg = seg_first + (int)blockIdx.y / H, b = blockIdx.z;
    const int t_begin = seg * seg_len;
    // Tokens past the chunks the segment's transition ran have w = 0 (it
    // stopped once M had decayed below fp32 resolution): nothing to add.
    const int t_end = min(min(T, t_begin + seg_len),
                          trans_len ? t_begin + abs(trans_len[((long)b * nseg + seg) * H + h]) * C : T);
    const int tile0 = blockIdx.x * CORR_TILES;
    if (t_begin + tile0 * C >= t_end) return;
    // Tile i's w into stage i & 1 (one commit group; rows past the segment zero).
    auto fetch = [&](int i) {
        const int t0 = t_begin + (tile0 + i) * C;
        if (i < CORR_TILES && t0 < t_end) {
            for (int idx = tid; idx < C * D / 8; idx += 256) {
                const int r = idx / (D / 8), q8 = 8 * (idx % (D / 8));
                __half* dst = &m.w[i & 1][r][q8];
                if (t0 + r < t_end) corr_cp16(dst, wbuf + (((long)b * T + t0 + r) * H + h) * D + q8);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    fetch(0);
    const float* src = seg_states + (((long)b * nseg + seg) * H + h) * (long)(D * D);
    for (int idx = tid; idx < D * D / 4; idx += 256) {
        const int r = idx / (D / 4), q4 = 4 * (idx % (D / 4));
        const float4 x = *reinterpret_cast<const float4*>(src + (long)r * D + q4);
        *reinterpret_cast<uint2*>(&m.s[r][q4]) = make_uint2(pack_f16x2(x.x, x.y), pack_f16x2(x.z, x.w));
    }
    const int rb = (warp >> 1) * 16, cb = (warp & 1) * 64;
    const int l = tid & 31, g = l >> 2, t4 = l & 3;
    for (int i = 0; i < CORR_TILES; ++i) {
        const int t0 = t_begin + (tile0 + i) * C;
        if (t0 >= t_end) break;
        fetch(i + 1);                                   // the other stage is free (barrier below)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncthreads();                                // tile i's w is in
        float2 ov[8][2];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int r = rb + g + 8 * e2;
                ov[j][e2] = make_float2(0.f, 0.f);
                if (t0 + r < t_end)
                    ov[j][e2] = *reinterpret_cast<const float2*>(out + (((long)b * T + t0 + r) * H + h) * D + cb + 8 * j + 2 * t4);
            }
        float acc[8][4];
        zero_acc(acc);
        wmm_f16_ah<8, D, true, D + 8, D + 8>(acc, rb, cb, &m.w[i & 1][0][0], &m.s[0][0]);
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
                const int r = rb + g + 8 * e2;
                if (t0 + r < t_end) {
                    float2* o = reinterpret_cast<float2*>(out + (((long)b * T + t0 + r) * H + h) * D + cb + 8 * j + 2 * t4);
                    *o = make_float2(ov[j][e2].x + acc[j][2 * e2], ov[j][e2].y + acc[j][2 * e2 + 1]);
                }
            }
        __syncthreads();                                // stage i & 1 is consumed
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Number of time segments per (batch, head).  Segmenting costs a second
// chunk recursion per segment (the transition), a combine and a correction,
// so it pays only when the (batch, head) pairs alone leave SMs idle.
// Automatic choice (requested == 0):
//  * kDecayRule (the transitions end once decayed, after a chunk or two with
//    decaying gates): one zero-start CTA per SM, n = #SMs / (B*H), from 32
//    chunks on, when n >= 3, or (scalar gate) n = 2 with at least 85% of the
//    SMs busy.  Measured on B200 against the prep pool (us): scalar gate,
//    T 8192, B*H = 48: n = 3 430, pool 556, n = 2 (96 SMs busy) 611;
//    B*H = 64, T 2048: n = 2 190, pool 213.  Per-channel gate: B*H = 48,
//    T 8192: n = 3 641, pool 697; B*H = 32, T 16384: n = 4 808, pool 1347;
//    B*H = 16, T 65536: n = 9 1551, n = 5 with full transitions 2443; but
//    B*H = 64, T 2048: n = 2 227-232, pool 225-229 (no gain: the pool keeps
//    per-channel gates at n = 2).
//  * kNoAllocRule (the fixed-scratch entry, whose transitions run in full
//    and whose segments need two states each): n = #SMs / (B*H) from
//    B*H*4 <= #SMs and 64 chunks on.
enum SegmentRule { kDecayRule, kNoAllocRule };
int choose_segments(int requested, int BH, int nchunks, SegmentRule rule, bool channel) {
    if (nchunks <= 1 || requested == 1) return 1;
    int n = requested;
    if (n <= 0) {
        const int sms = sm_count();
        n = sms / BH;
        if (rule == kDecayRule) {
            if (nchunks < 32 || n < 2) return 1;
            if (n == 2 && (channel || 2 * BH * 100 < 85 * sms)) return 1;
        } else if (nchunks < 64 || n < 4) {
            return 1;
        }
    }
    return n < nchunks ? n : nchunks;
}

template <bool CHANNEL>
cudaError_t launch(const Problem& p, cudaStream_t stream) {
    cudaError_t ea = set_smem_limit(reinterpret_cast<const void*>(chunk_fwd_kernel<CHANNEL>), SMEM_BYTES);
    if (ea != cudaSuccess) return ea;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, p.q, p.H, p.T, p.B) || !make_map(&mk, p.k, p.H, p.T, p.B) ||
        !make_map(&mv, p.v, p.H, p.T, p.B) || !make_out_map(&mo, p.out, p.H, p.T, p.B))
        return cudaErrorInvalidValue;
    float* out = static_cast<float*>(p.out);
    const int nchunks = (p.T + C - 1) / C;
    int nseg = choose_segments(p.segments, p.B * p.H, nchunks, kDecayRule, CHANNEL);
    auto unsegmented = [&]() -> cudaError_t {
        // Chunk-local work and the state chain on different SMs when two per
        // (batch, head) fit: by default one prep pool over all SMs; a cluster
        // per pair with GDN_CHUNK_KERNEL=pair, one CTA per pair with =single
        // (tests, tuning).
        const char* force = getenv("GDN_CHUNK_KERNEL");
        const bool split = force ? (strcmp(force, "pair") == 0 || strcmp(force, "pool") == 0)
                                 : (2 * p.B * p.H <= sm_count());
        const bool pool = !force || strcmp(force, "pool") == 0;
        if (split) {
            cudaError_t e = launch_chunk_pair_sm100(p, stream, pool ? sm_count() : 0);
            if (pool && e == cudaErrorMemoryAllocation) {
                // No room for the pool's task records (nothing was launched):
                // the cluster form needs no scratch.  The failed allocation
                // is the pending error, if any, that is cleared here.
                if (cudaPeekAtLastError() == cudaErrorMemoryAllocation) (void)cudaGetLastError();
                e = launch_chunk_pair_sm100(p, stream, 0);
            }
            return e;
        }
        Params prm{p.g, p.beta, p.state_in, p.state_out, nullptr, out, p.T, p.H, p.B,
                   1, nchunks * C, 1, 1};
        chunk_fwd_kernel<CHANNEL><<<p.B * p.H, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mo, prm);
        return cudaGetLastError();
    };
    if (nseg <= 1) return unsegmented();
    // Segment-parallel path in two chunk passes.  One launch runs segment 0
    // from the true initial state and every other segment from a zero state,
    // writing outputs and end states, and, in a second set of CTAs, the
    // transitions M of segments 1 .. n-1 with v = 0 from the identity,
    // writing w_t = M_t^T q_t per token (fp16).  A serial combine turns the
    // end states into true start states; the correction then adds
    // S_start^T w_t to the outputs of segments 1 .. n-1 (the state map is
    // affine: S_t = M_t S_start + S_t(0)).
    const int seg_len = ((nchunks + nseg - 1) / nseg) * C;
    nseg = (p.T + seg_len - 1) / seg_len;
    const size_t slab = (size_t)p.B * nseg * p.H * D * D;
    const size_t wlen = (size_t)p.B * p.T * p.H * D;
    float* ws = nullptr;
    const size_t nlen = ((size_t)p.B * nseg * p.H + 3) / 4 * 4;   // ints, 16-byte multiple
    cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&ws),
                                    2 * slab * sizeof(float) + nlen * sizeof(int) + wlen * sizeof(__half),
                                    stream);
    if (e == cudaErrorMemoryAllocation && p.segments == 0) {
        // An automatic choice whose scratch cannot be had (nothing was
        // launched): the unsegmented path, whose own fallback needs none.
        if (cudaPeekAtLastError() == cudaErrorMemoryAllocation) (void)cudaGetLastError();
        return unsegmented();
    }
    if (e != cudaSuccess) return e;
    float* seg_states = ws;
    float* trans = ws + slab;
    int* trans_len = reinterpret_cast<int*>(ws + 2 * slab);
    __half* wbuf = reinterpret_cast<__half*>(trans_len + nlen);
    CUtensorMap mw;
    if (!make_half_map(&mw, wbuf, p.H, p.T, p.B)) {
        const cudaError_t ef = cudaFreeAsync(ws, stream);
        return ef != cudaSuccess ? ef : cudaErrorInvalidValue;
    }
    Params p1{p.g, p.beta, p.state_in, seg_states, trans, out, p.T, p.H, p.B, nseg, seg_len, 1, nseg};
    p1.wout = wbuf;
    p1.trans_first = 1;
    p1.in_first_only = true;
    p1.trans_len = trans_len;
    chunk_fwd_kernel<CHANNEL><<<p.B * (2 * nseg - 1) * p.H, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mw, p1);
    e = cudaGetLastError();
    if (e == cudaSuccess) {
        combine_segments_kernel<<<p.B * p.H * (D / CB_COLS), 256, 0, stream>>>(
            seg_states, trans, p.state_in, p.state_out, p.H, nseg, 1, trans_len);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        e = set_smem_limit(reinterpret_cast<const void*>(segment_correction_kernel), (int)sizeof(CorrSmem));
        if (e == cudaSuccess) {
            const int groups = (seg_len / C + CORR_TILES - 1) / CORR_TILES;
            segment_correction_kernel<<<dim3(groups, (nseg - 1) * p.H, p.B), 256, sizeof(CorrSmem), stream>>>(
                seg_states, wbuf, out, p.T, p.H, nseg, seg_len, 1, trans_len);
            e = cudaGetLastError();
        }
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : ef;
}

// ---- no-allocation variant of the segment-parallel path ---------------------
// Scratch for callers that must not allocate: a fixed array in the library's
// device image (every GPU that loads the library holds it until exit).
// Host code may not use the array's name as a device address; the address is
// looked up with cudaGetSymbolAddress once per device (see below).
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

cudaError_t noalloc_scratch_address(float** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    constexpr int kMaxDevices = 128;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    static std::mutex mu;
    static float* addr[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {   // first call on this device, device current
        void* a = nullptr;
        e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<float*>(a);
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

template <bool CHANNEL>
cudaError_t launch_noalloc(const Problem& p, cudaStream_t stream, bool* over_limit) {
    *over_limit = false;
    const int nchunks = (p.T + C - 1) / C;
    int nseg = choose_segments(p.segments, p.B * p.H, nchunks, kNoAllocRule, CHANNEL);
    const int seg_len = ((nchunks + nseg - 1) / nseg) * C;
    if (nseg > 1) nseg = (p.T + seg_len - 1) / seg_len;
    const size_t slab = (size_t)p.B * nseg * p.H * D * D;
    if (nseg > 1 && 2 * slab > kNoAllocScratchFloats) {
        *over_limit = true;          // rejected before anything is launched
        return cudaErrorInvalidValue;
    }
    cudaError_t ea = set_smem_limit(reinterpret_cast<const void*>(chunk_fwd_kernel<CHANNEL>), SMEM_BYTES);
    if (ea != cudaSuccess) return ea;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, p.q, p.H, p.T, p.B) || !make_map(&mk, p.k, p.H, p.T, p.B) ||
        !make_map(&mv, p.v, p.H, p.T, p.B) || !make_out_map(&mo, p.out, p.H, p.T, p.B))
        return cudaErrorInvalidValue;
    float* out = static_cast<float*>(p.out);
    if (nseg <= 1) {
        Params prm{p.g, p.beta, p.state_in, p.state_out, nullptr, out, p.T, p.H, p.B,
                   1, nchunks * C, 1, 1};
        chunk_fwd_kernel<CHANNEL><<<p.B * p.H, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mo, prm);
        return cudaGetLastError();
    }
    float* ws = nullptr;
    cudaError_t e = noalloc_scratch_address(&ws);
    if (e != cudaSuccess) return e;
    // Every scratch element read below is written earlier in this call (pass
    // 1 writes all end states and transitions), so nothing is cleared.
    float* seg_states = ws;
    float* trans = ws + slab;
    Params p1{p.g, p.beta, nullptr, seg_states, trans, nullptr, p.T, p.H, p.B, nseg, seg_len, 1, nseg};
    chunk_fwd_kernel<CHANNEL><<<2 * p.B * nseg * p.H, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mo, p1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    combine_segments_kernel<<<p.B * p.H * (D / CB_COLS), 256, 0, stream>>>(
        seg_states, trans, p.state_in, p.state_out, p.H, nseg, 0, nullptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Params p2{p.g, p.beta, seg_states, nullptr, nullptr, out, p.T, p.H, p.B, nseg, seg_len, nseg, 1};
    chunk_fwd_kernel<CHANNEL><<<p.B * nseg * p.H, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mo, p2);
    return cudaGetLastError();
}

}  // namespace

// Stream-ordered workspace from a memory pool owned by this library, one per
// device, that keeps its memory between calls (release threshold: no limit).
// The device's default pool returns its memory to the system at every
// synchronisation unless its owner configured it otherwise, and mapping it
// again on the next call cost milliseconds.  Held: the largest workspace in
// use at once.
cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
    // Test hook: scratch that cannot be had, as on a full device (nothing is
    // allocated or launched).  Unset in normal use.
    if (getenv("GDN_TEST_FAIL_WORKSPACE")) return cudaErrorMemoryAllocation;
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!pools[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t pool = nullptr;
            e = cudaMemPoolCreate(&pool, &props);
            if (e != cudaSuccess) return e;
            cuuint64_t keep = ~cuuint64_t(0);
            e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
            if (e != cudaSuccess) {
                cudaMemPoolDestroy(pool);
                return e;
            }
            pools[dev] = pool;
        }
    }
    return cudaMallocFromPoolAsync(ptr, bytes, pools[dev], stream);
}

cudaError_t set_smem_limit(const void* kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, int> done;
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find({dev, kernel});
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[{dev, kernel}] = bytes;
    return e;
}

int sm_count() {
    constexpr int kMaxDevices = 128;
    static std::mutex mu;
    static int n[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (n[dev] == 0) {
        int c = 0;
        n[dev] = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && c > 0
                     ? c : 148;
    }
    return n[dev];
}

cudaError_t launch_chunk_sm100_noalloc(const Problem& p, cudaStream_t stream, bool* over_limit) {
    *over_limit = false;
    if (p.io_f32 || !p.out_f32 || p.dk != D || p.dv != D) return cudaErrorNotSupported;
    return p.per_channel ? launch_noalloc<true>(p, stream, over_limit)
                         : launch_noalloc<false>(p, stream, over_limit);
}

cudaError_t launch_chunk_sm100(const Problem& p, cudaStream_t stream) {
    if (p.io_f32 || !p.out_f32 || p.dk != D || p.dv != D) return cudaErrorNotSupported;
    return p.per_channel ? launch<true>(p, stream) : launch<false>(p, stream);
}

cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_status_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    unsigned int pair_status = 0;
    e = read_and_clear_pair_status(&pair_status);
    *status |= pair_status;
    return e;
}

}  // namespace gdn
