// chunk_pair_sm100.cu -- chunkwise prefill with the work of one (batch, head)
// split between a "prep" CTA and a "chain" CTA on two SMs.
//
// Same chunk algebra as chunk_sm100.cu (Atomic-GDN2 model card, section 2.1;
// chunkwise mode of the "Gated DeltaNet" entity trail, finding of
// 2026-07-29):
//   A_rj = b_r k_r^T Diag(exp(G_r - G_j)) k_j (j < r),  T' = (I + A)^{-1} Diag(b)
//   P_rj = q_r^T Diag(exp(G_r - G_j)) k_j (j <= r)
//   U = T' V - T' (K * E) S,  O = (Q * E) S + P U,  S <- Diag(E_last) S + (K * D)^T U
// A, P and T' depend on the chunk's own inputs only; U, O and the new S
// depend on the state.  The two halves run on different SMs and overlap
// (roles as in the cluster form; the pool form below moves the chain's
// operand build to the prep side):
//
//   CTA 0 ("prep"):  gate prep, X = [K*F; Q*F](K/F)^T on tcgen05, A and P,
//                    the fp32 triangular solve, T' and P as bf16 hi + lo;
//                    hands the 32 KB of T' and P to CTA 1 with a bulk copy
//                    into CTA 1's shared memory (no multicast), then moves on
//                    to the next chunk.
//   CTA 1 ("chain"): owns the fp32 state; gate prep for E and D, the derived
//                    operands K*E, Q*E, K*D, and the state-dependent products
//                    W^T, U^T, O^T and SN; writes the outputs.
//
// Two launch forms share the code of both roles:
//
// chunk_pair_kernel, a cluster of two CTAs per (batch, head).  Hand-off: CTA
//   1's "full" mbarrier (armed by CTA 0 with a remote arrive.expect_tx,
//   completed by the bulk copy's byte count) and CTA 0's "empty" mbarrier (a
//   remote arrive from CTA 1 once the products that read the slot are
//   complete).  CTA 0 therefore works on chunk c + 1 while CTA 1 works on
//   chunk c.
//
// chunk_pool_kernel, a cooperative grid of one CTA per SM: B*H chain CTAs and
//   every other SM a prep CTA.  The prep CTAs share the (batch, head, chunk)
//   tasks, chunk-major (task i: chunk i / (B*H), pair i % (B*H); CTA j takes
//   tasks j, j + n_prep, ...).  Each writes its task's record to a global
//   buffer: T' (or, with per-channel gates, T and beta), P, and the chain's
//   operands K*E, Q*E, K*D and exp(G_last), as images of the chain's
//   shared-memory tiles; then it sets the task's flag (release).  A chain
//   tries the flag of its next chunk early (acquire), prefetches the record
//   into L2, and fetches it in three bulk copies, each as soon as the
//   previous chunk's products that read the same tiles are complete.  It
//   discards each record from L2 after its last read.  With more prep CTAs
//   than chains, no chain waits on a single prep CTA, the SMs that a cluster
//   per pair leaves idle do prep work, and the chain needs no raw K, Q or
//   gate.
//
// Every wait is bounded (kWaitBudgetNs); on expiry a CTA records it in its
// status word, stops, drains its own copies and returns.
//
// Precision and operand formats are those of chunk_sm100.cu (bf16 hi + lo for
// the factored A/P operands, T', P, U and K*D; fp16 for S, W and Q*E; fp32
// accumulation in TMEM; fp32 output).

#include <cuda.h>
#include <cudaTypedefs.h>

#include "chunk_common.cuh"
#include "gdn_internal.cuh"
#include "prologue_math.cuh"
#include "sm100_util.cuh"

#include <cstdlib>

namespace gdn {

__device__ unsigned int g_pair_status_word = 0;

namespace {

using namespace sm100;
using namespace chunk;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 256;

// ---- CTA 0 (prep) shared memory -----------------------------------------------
constexpr uint32_t P_IN = 0;                  // 32 KB raw K, Q [half][K 64 | Q 64][128 B]
constexpr uint32_t P_X = 32768;               // 112 KB:
constexpr uint32_t P_AH = P_X;                //   X operands (per-channel): 32 KB
constexpr uint32_t P_AL = P_X + 32768;        //   32 KB
// B operand of X, [64-channel half][hi rows 0-95 | lo rows 0-95][128 B]:
// rows 0-31 = K/F of tokens 0-31 (reference 15), rows 32-95 = K*exp(G_47 - G)
// of tokens 0-63, so that one N = 96 product per k-step covers both; hi and
// lo back to back make [hi; lo] one N = 192 operand (A hi times both in one
// product, see the X issue).
constexpr uint32_t P_CB = P_X + 65536;        //   48 KB
constexpr uint32_t CB_HALF = 96 * 128;        //   one of hi / lo of one channel half
constexpr uint32_t P_A = P_X + 32768;         //   16 KB A fp32 (fidx layout)
constexpr uint32_t P_T = P_X + 49152;         //   16 KB T fp32 (tidx layout)
constexpr uint32_t P_Y = P_X + 65536;         //   10 KB solve scratch 2 x [32][40]
constexpr uint32_t P_SMALL = P_X + 114688;
constexpr uint32_t P_GAM = P_SMALL;           // 64 f32
constexpr uint32_t P_BETA = P_GAM + 256;      // 64 f32
constexpr uint32_t P_REF0 = P_BETA + 256;     // 128 f32
constexpr uint32_t P_REF1 = P_REF0 + 512;     // 128 f32
constexpr uint32_t P_ER = P_REF1 + 512;       // 64 f32: exp(G_r - G_31)  (scalar gate)
constexpr uint32_t P_FJ = P_ER + 256;         // 64 f32: exp(G_31 - G_j)
constexpr uint32_t P_SAFE = P_FJ + 256;       // int: product form in range
constexpr uint32_t P_BAR = P_SAFE + 16;       // tma, mma, empty, g
constexpr uint32_t P_TMEM = P_BAR + 32;
// T' hi, T' lo, P hi, P lo (4 x 8 KB) for the bulk copy to CTA 1; apart from
// the X region so that the copy of chunk c overlaps the X build of chunk c + 1.
constexpr uint32_t P_LAST = P_TMEM + 16;      // 128 f32: G of the chunk's last token (pool form)
constexpr uint32_t P_STAGE = (P_LAST + 512 + 1023) / 1024 * 1024;
// Per-channel g of the next chunk, by TMA: four [64 tokens][32 channels] fp32
// boxes, 128-byte swizzled (8 KB each).
constexpr uint32_t P_G = P_STAGE + 32768;
constexpr uint32_t P_USED = P_G + 32768;
// Pool form, scalar gate: K*E bf16 [half][64 r][128 B] for the prep's own
// W^T product (the per-channel X operands' space, unused with a scalar gate).
constexpr uint32_t P_KE = P_X;
// Fused prologue, prep CTA, before the X operands are built (same space):
// q and k history rows [2][3][128] fp32, taps of q | k [256] float4, and the
// per-channel-chunk sums of squares [16][64] fp32.
constexpr uint32_t P_PH = P_X;
constexpr uint32_t P_PW = P_X + 3072;
constexpr uint32_t P_PS = P_X + 7168;

// ---- CTA 1 (chain) shared memory ----------------------------------------------
constexpr uint32_t C_IN = 0;                  // 32 KB raw K, Q
constexpr uint32_t C_V = 32768;               // 16 KB raw V
constexpr uint32_t C_S = 49152;               // 32 KB S fp16 [j half][128 i][64 j]
constexpr uint32_t C_KE = 81920;              // 16 KB K*E bf16; then W^T fp16 [128 i][64 r]
constexpr uint32_t C_QE = 98304;              // 16 KB Q*E fp16
constexpr uint32_t C_KDH = 114688;            // 16 KB K*D bf16 hi
constexpr uint32_t C_KDL = 131072;            // 16 KB K*D bf16 lo
constexpr uint32_t C_UH = 147456;             // 16 KB U^T hi [128 j][64 r]
constexpr uint32_t C_UL = 163840;             // 16 KB U^T lo
constexpr uint32_t C_OST = C_UH;              // after O: 32 KB O fp32 [64 t][128 j] for the TMA store
constexpr uint32_t C_SLOT = 180224;           // 32 KB T' hi, T' lo, P hi, P lo (from CTA 0)
constexpr uint32_t C_TH = C_SLOT, C_TL = C_SLOT + 8192, C_PH = C_SLOT + 16384, C_PL = C_SLOT + 24576;
constexpr uint32_t C_SMALL = C_SLOT + 32768;
constexpr uint32_t C_GAM = C_SMALL;           // 64 f32
constexpr uint32_t C_LAST = C_GAM + 256;      // 128 f32
constexpr uint32_t C_BAR = C_LAST + 512;      // tma_kq, tma_v, mma, full, out, full_b, full_c
constexpr uint32_t C_TMEM = C_BAR + 56;
constexpr uint32_t C_FETCHED = C_TMEM + 8;    // 3 int: record parts fetched (pool form)
constexpr uint32_t C_USED_BASE = C_FETCHED + 16;
// Fused prologue (pool form): v's history rows [3][128] fp32 and taps [128] float4.
constexpr uint32_t C_HV = C_USED_BASE;
constexpr uint32_t C_TV = C_HV + 1536;
constexpr uint32_t C_USED = C_TV + 2048;

constexpr uint32_t SLOT_BYTES = 32768;

// Pool form: task records kept per (batch, head) at once (a ring; >= 4 for
// progress, see PairParams), and the scratch the records may take before the
// ring is shortened to kPoolRing slots.
constexpr int kPoolRing = 8;
constexpr size_t kPoolScratchBytes = size_t(256) << 20;
static_assert(kPoolRing >= 4, "the record ring needs at least 4 slots");

// Pool form: one task's record in the global buffer, in three parts that the
// chain fetches apart, each as soon as the previous chunk's products that read
// the same shared-memory tiles are complete.  Tiles are the images of the
// chain's shared-memory tiles (same swizzle), so each part is a plain copy.
// With per-channel gates the prep CTAs bound the launch, so part A carries T
// itself (fp32, as the solve leaves it) and beta, and the chain forms T' =
// T Diag(beta) as bf16 hi + lo; with a scalar gate it carries T'.
constexpr uint32_t TA_T = 0;                  // part A: T' hi, T' lo, or T fp32 (16 KB)
constexpr uint32_t TA_KE = 16384;             //         K*E bf16 (16 KB)
constexpr uint32_t TB_QE = 32768;             // part B: Q*E fp16 (16 KB)
constexpr uint32_t TC_P = 49152;              // part C: P hi, P lo (16 KB)
constexpr uint32_t TC_KD = 65536;             //         K*D bf16 hi, lo (32 KB)
constexpr uint32_t TC_EL = 98304;             //         exp(G_last) per channel (512 B)
constexpr uint32_t TA_BETA = 98816;           // part A: beta (256 B; per-channel gates)
constexpr uint32_t TASK_BYTES = 99072;         // 774 lines of 128 bytes
static_assert(TASK_BYTES % 128 == 0, "records are whole L2 lines (discarded after use)");
constexpr uint32_t PART_A = TB_QE - TA_T, PART_B = TC_P - TB_QE, PART_C = TA_BETA - TC_P;
constexpr uint32_t SMEM_BYTES = (P_USED > C_USED ? P_USED : C_USED) + 1024;

// TMEM columns.  CTA 0: X (128 rows x up to 96).  CTA 1: W^T, U^T, O^T, SN.
constexpr uint32_t TM_X = 0;
constexpr uint32_t TM_WT = 0, TM_UT = 64, TM_OT = 128, TM_SN = 256;

struct PairParams {
    const float* g;            // [B, T, H] or [B, T, H, D]
    const float* beta;         // [B, T, H]
    const float* state_in;     // [B, H, D, D] or null
    float* state_out;          // [B, H, D, D] or null
    float* out;                // [B, T, H, D] fp32
    int T, H, B;
    // Pool form: a ring of `ring` task records per (batch, head); record
    // slot c % ring holds chunk c.  flags[pair][slot] = c + 1 once chunk c's
    // record is stored (release); consumed[pair] = n once the chain has read
    // (and discarded from L2) the records of chunks 0 .. n - 1, so a prep CTA
    // may rewrite slot c % ring when consumed >= c - ring + 1.  All zero at
    // launch.  The chain publishes consumed = c - 1 while it works on chunk
    // c + 1 (it has read chunk c - 1's record by then).  With ring >= 4 this
    // cannot deadlock: a prep CTA publishes its finished record before it
    // waits for a slot, so every task of lower index than the unfinished one
    // of lowest index (chunk-major order) has its record published, and that
    // task waits only for its chain to reach chunk c - ring + 2, which needs
    // records of lower index only.
    uint8_t* slots;            // [B*H][ring][TASK_BYTES]
    unsigned int* flags;       // [B*H][ring]
    unsigned int* consumed;    // [B*H]
    int ring;
    // Failure-detection test hooks (pool form): the budget of a chain's wait
    // for a record's flag, and one task whose flag is never set (-1: none).
    // A chain that waits for that flag gives up when the budget runs out,
    // records the timeout in the status word and returns; prep CTAs never
    // wait for chains, so the launch still ends.
    unsigned long long flag_budget_ns;
    long long withheld_task;
    // Fused input prologue (pool form with PRO): the tensor maps and g, beta
    // point at the layer's raw projections, and the kernel applies the width-4
    // causal convolution (history from the ring), the activation, the q/k L2
    // norm and the gate maps while loading them, as gdn_prologue would.
    const float* conv_w = nullptr;          // [H, 3D, 4], channels q | k | v
    const float* conv_ring = nullptr;       // [B, H, 4, 3D] or null: history ring
    const int* pos0 = nullptr;              // [B] or null (0)
    const __nv_bfloat16* q_raw = nullptr;   // [B, T, H, D]: history rows
    const __nv_bfloat16* k_raw = nullptr;
    const __nv_bfloat16* v_raw = nullptr;
    bool silu = true;
};

// Fused prologue: one 64-token tile of one tensor (bf16, TMA layout: halves
// of 64 channels `half_stride` bytes apart, [64 tokens][128 B], 128-byte
// swizzle) becomes the recurrence's input in place: the width-4 causal
// convolution (tap 3 on the current token; `hist` [3][128] fp32 holds the
// three tokens before the tile), the activation, the L2 norm over the 128
// channels when `norm` (x (sum x^2 + 1e-6)^-1/2), bf16 rounding; rows at or
// past `nvalid` become zero.  Thread t of 256 takes channels 2 (t & 63) and
// 2 (t & 63) + 1 over tokens 16 (t >> 6) .. + 15, the tap window sliding in
// registers; a token's sum of squares is the butterfly total of its block's
// two warps (`ss` 8 x 16 fp32 of shared scratch).  With keep_last, the raw
// tokens 61-63 replace `hist` (the next consecutive tile's history).  Ends
// with a proxy fence and a barrier (the tensor core may read the tile next).
__device__ __forceinline__ void pro_convert_tile(uint8_t* tile, uint32_t half_stride, float* hist,
                                                 const float4* taps, float* ss, int nvalid, bool silu,
                                                 bool norm, bool keep_last, int tid) {
    using namespace prologue_math;
    const int cp = tid & 63, blk = tid >> 6, lane = tid & 31, warp = tid >> 5;
    const int c = 2 * cp;
    uint8_t* col = tile + (c >> 6) * half_stride + ((c & 7) << 1);
    const uint32_t chunk = (c & 63) >> 3;
    const float4 w0 = taps[c], w1 = taps[c + 1];
    const float2 ta = make_float2(w0.x, w1.x), tb = make_float2(w0.y, w1.y);
    const float2 tc = make_float2(w0.z, w1.z), td = make_float2(w0.w, w1.w);
    const int r0 = 16 * blk;
    auto row = [&](int r) -> float2 {
        if (r >= 0) return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(col + swz(r, chunk)));
        return make_float2(hist[(3 + r) * D + c], hist[(3 + r) * D + c + 1]);
    };
    float2 win[3] = {row(r0 - 3), row(r0 - 2), row(r0 - 1)};
    float2 y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 x = row(r0 + i);
        const float2 a = fma2(ta, win[0], fma2(tb, win[1], fma2(tc, win[2], mul2(td, x))));
        y[i] = r0 + i < nvalid ? act_fn2(a, silu) : make_float2(0.f, 0.f);
        win[0] = win[1]; win[1] = win[2]; win[2] = x;
    }
    if (norm) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = fmaf(y[i].x, y[i].x, y[i].y * y[i].y);
        butterfly_sums16(v, lane);
        if ((lane & 1) == 0) ss[warp * 16 + butterfly_token(lane)] = v[0];
    }
    __syncthreads();                          // every raw row read; the sums in
    // Lane l computes the inverse norm of token r0 + (l & 15) once; row i
    // takes it from lane i.
    float inv_l = 1.f;
    if (norm) inv_l = rsqrtf(ss[(2 * blk) * 16 + (lane & 15)] + ss[(2 * blk + 1) * 16 + (lane & 15)] + 1e-6f);
    if (keep_last && blk == 3) {              // raw tokens 61-63: the next tile's history
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            hist[i * D + c] = win[i].x;
            hist[i * D + c + 1] = win[i].y;
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float2 o = y[i];
        if (norm) {
            const float inv = __shfl_sync(0xffffffffu, inv_l, i);
            o.x *= inv; o.y *= inv;
        }
        *reinterpret_cast<__nv_bfloat162*>(col + swz(r0 + i, chunk)) = __floats2bfloat162_rn(o.x, o.y);
    }
    fence_async_smem();
    __syncthreads();
}

template <bool CHANNEL, bool POOL, bool PRO = false>
__device__ __forceinline__ void pair_body(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                          const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                                          const CUtensorMap& tm_g, const PairParams& p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int T = p.T;
    const int H = p.H;
    const int nbh = p.B * H;
    // Role: rank 0 = prep, 1 = chain.  Pool form: CTAs 0 .. B*H-1 are the
    // chains (one per pair), the rest prep CTAs.
    const uint32_t rank = POOL ? ((int)blockIdx.x < nbh ? 1u : 0u) : cluster_ctarank();
    const int pair = POOL ? (rank ? (int)blockIdx.x : 0) : (int)(blockIdx.x >> 1);
    const int h = pair % H;
    const int b = pair / H;
    const int nchunks = (T + C - 1) / C;
    // Gate-prep / tile-building ownership (see chunk_sm100.cu): channel chunk
    // ck of 8 channels, lane tg owns tokens tg + 16 u.
    const int ck = 2 * warp + (lane >> 4);
    const int tg = lane & 15;
    const int ckh = ck >> 3;
    const int ckc = ck & 7;
    bool ok = true;

    // Both CTAs: barriers and TMEM, then a cluster barrier so that no remote
    // arrive or copy can reach an uninitialised barrier.
    const uint32_t bar0 = sbase + (rank == 0 ? P_BAR : C_BAR);
    if (tid == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        if (rank == 1) {
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_o);
        }
        if (rank == 0 && CHANNEL) prefetch_tensormap(&tm_g);
        for (int i = 0; i < (rank == 0 ? 4 : 7); ++i) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
    }
    const uint32_t tmem_cols = rank == 0 ? 256 : 512;   // prep: X with its hi / lo halves
    if (warp == 0) {
        tmem_alloc(sbase + (rank == 0 ? P_TMEM : C_TMEM), tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t*>(smem + (rank == 0 ? P_TMEM : C_TMEM));
    if (!POOL) cluster_sync();

    uint32_t mma_phase = 0;
    auto mma_sync = [&]() {
        ok = ok && mbar_wait(bar0 + 8 * (rank == 0 ? 1 : 2), mma_phase, &g_pair_status_word);
        mma_phase ^= 1;
        tc_fence_after();
    };

    // Per-channel cumulative log-decay of this thread's 4 tokens x 8 channels
    // (registers); block references / last token stored by lane tg = 15.
    // Loads are issued one chunk ahead (gate_load for chunk c + 1 once chunk c
    // no longer needs its own values), so their latency is hidden behind the
    // rest of the chunk; the scan (gate_channel) runs at the start of the
    // chunk.  They are issued after a proxy fence, not before one: the fence
    // waits for the thread's outstanding loads (measured on B200).
    auto gate_load = [&](int chunk, float (&gam)[4][8]) {
        const int t0 = chunk * C;
        const long tk0 = ((long)b * T + t0) * H + h;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = tg + 16 * u;
            if (t0 + r < T) {
                const float4* src = reinterpret_cast<const float4*>(p.g + (tk0 + (long)r * H) * D + 8 * ck);
                const float4 a = src[0], c = src[1];
                gam[u][0] = a.x; gam[u][1] = a.y; gam[u][2] = a.z; gam[u][3] = a.w;
                gam[u][4] = c.x; gam[u][5] = c.y; gam[u][6] = c.z; gam[u][7] = c.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gam[u][e] = 0.f;
            }
        }
    };
    auto gate_scan = [&](float (&gam)[4][8], float* ref0, float* ref1, float* last) {
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
        if (tg == 15) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (ref0) ref0[8 * ck + e] = gam[0][e];
                if (ref1) ref1[8 * ck + e] = gam[2][e];
                if (last) last[8 * ck + e] = gam[3][e];
            }
        }
    };
    auto gate_channel = [&](int t0, long tk0, float (&gam)[4][8], float* ref0, float* ref1,
                            float* last) {
        if (t0 + 2 * C < T) {     // warm L2 two chunks ahead
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = 2 * C + tg + 16 * u;
                if (t0 + r < T) prefetch_l2(p.g + (tk0 + (long)r * H) * D + 8 * ck);
            }
        }
        gate_scan(gam, ref0, ref1, last);
    };
    // Scalar gate and beta, warp 0: lane holds tokens lane and 32 + lane.
    // gate_scalar_load reads them into registers; gate_scalar scans g into
    // sGam (and stores beta when sBeta is given).
    auto gate_scalar_load = [&](int bb, int hh, int chunk, bool with_beta, float (&bg)[4]) {
        bg[0] = bg[1] = bg[2] = bg[3] = 0.f;
        if (warp != 0) return;
        const int t0 = chunk * C;
        const long tk0 = ((long)bb * T + t0) * H + hh;
        if (t0 + lane < T) {
            if (with_beta) bg[0] = p.beta[tk0 + (long)lane * H];
            if (!CHANNEL) bg[2] = p.g[tk0 + (long)lane * H];
        }
        if (t0 + 32 + lane < T) {
            if (with_beta) bg[1] = p.beta[tk0 + (long)(32 + lane) * H];
            if (!CHANNEL) bg[3] = p.g[tk0 + (long)(32 + lane) * H];
        }
        if (PRO) {   // raw projections: beta = sigmoid, g = -min(softplus, 5); padding stays 0
            using namespace prologue_math;
            if (t0 + lane < T) {
                if (with_beta) bg[0] = sigmoid_fn(bg[0]);
                if (!CHANNEL) bg[2] = gate_fn(bg[2]);
            }
            if (t0 + 32 + lane < T) {
                if (with_beta) bg[1] = sigmoid_fn(bg[1]);
                if (!CHANNEL) bg[3] = gate_fn(bg[3]);
            }
        }
    };
    auto gate_scalar = [&](const float (&bg)[4], float* sGam, float* sBeta, float* sEr = nullptr,
                           float* sFj = nullptr, int* sSafe = nullptr) {
        if (warp != 0) return;
        const float b0 = bg[0], b1 = bg[1];
        float g0 = bg[2], g1 = bg[3];
        if (sBeta) {
            sBeta[lane] = b0;
            sBeta[32 + lane] = b1;
        }
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
            if (sEr) {
                // exp(G_r - G_j) = exp(G_r - G_31) exp(G_31 - G_j), exact in fp32
                // while the chunk's total decay is at most 80 (both factors
                // within exp(+-80)); otherwise the epilogue exponentiates directly.
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
    };

    if (rank == 0) {
        // =========================================================== prep CTA ===
        float* sGam = reinterpret_cast<float*>(smem + P_GAM);
        float* sBeta = reinterpret_cast<float*>(smem + P_BETA);
        float* sRef0 = reinterpret_cast<float*>(smem + P_REF0);
        float* sRef1 = reinterpret_cast<float*>(smem + P_REF1);
        float* sEr = reinterpret_cast<float*>(smem + P_ER);
        float* sFj = reinterpret_cast<float*>(smem + P_FJ);
        int* sSafe = reinterpret_cast<int*>(smem + P_SAFE);
        float* sA = reinterpret_cast<float*>(smem + P_A);
        float* sT = reinterpret_cast<float*>(smem + P_T);
        float* sY = reinterpret_cast<float*>(smem + P_Y);
        float* sLastP = reinterpret_cast<float*>(smem + P_LAST);
        const uint32_t bar_tma = sbase + P_BAR, bar_empty = sbase + P_BAR + 16;
        const uint32_t bar_g = sbase + P_BAR + 24;
        // Cluster form: CTA 1's slot and "full" barrier, as cluster addresses.
        const uint32_t peer_slot = POOL ? 0u : mapa_shared(sbase + C_SLOT, 1);
        const uint32_t peer_full = POOL ? 0u : mapa_shared(sbase + C_BAR + 24, 1);
        // The items this CTA prepares, in order: the chunks of its pair
        // (cluster form) or its share of the chunk-major task list (pool).
        const int nprep = POOL ? (int)gridDim.x - nbh : 1;
        const int pid = POOL ? (int)blockIdx.x - nbh : 0;
        const int ntasks = nbh * nchunks;
        const int nitems = POOL ? (pid < ntasks ? (ntasks - pid + nprep - 1) / nprep : 0) : nchunks;
        auto item = [&](int j, int& ib, int& ih, int& ic) {
            if (POOL) {
                const int task = pid + j * nprep;
                ic = task / nbh;
                const int pr = task - ic * nbh;
                ib = pr / H;
                ih = pr - ib * H;
            } else {
                ib = b; ih = h; ic = j;
            }
        };
        int kq_issued = 0;                    // K, Q loads issued (tid 0), for the drain
        auto item_valid = [&](int j) {   // tokens of item j's chunk inside the sequence
            int ib, ih, ic;
            item(j, ib, ih, ic);
            return T - ic * C < C ? T - ic * C : C;
        };
        // Fused prologue: item j's history rows (tokens t0-3 .. t0-1 of q and
        // k: thread tid takes channel tid & 127 of q (tid < 128) or k, from
        // the raw inputs, or from the ring before the first token) and the
        // taps of conv channel tid (q | k), into registers one item ahead.
        float hq[3] = {0.f, 0.f, 0.f};
        float4 tq = make_float4(0.f, 0.f, 0.f, 0.f);
        auto pro_load = [&](int j) {
            if (!PRO) return;
            int ib, ih, ic;
            item(j, ib, ih, ic);
            const int tn = tid >> 7, ch = tid & 127;
            const __nv_bfloat16* raw = tn == 0 ? p.q_raw : p.k_raw;
            const int p0 = p.pos0 ? p.pos0[ib] : 0;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const int t = ic * C - 3 + i;
                float x = 0.f;
                if (t >= 0) {
                    x = __bfloat162float(raw[(((long)ib * T + t) * H + ih) * D + ch]);
                } else if (p.conv_ring && p0 + t >= 0) {
                    x = p.conv_ring[(((long)ib * H + ih) * 4 + ((p0 + t) & 3)) * (3 * D) + tn * D + ch];
                }
                hq[i] = x;
            }
            tq = *reinterpret_cast<const float4*>(p.conv_w + ((long)ih * 3 * D + tid) * 4);
        };
        auto issue_kq = [&](int j) {
            int ib, ih, ic;
            item(j, ib, ih, ic);
            ++kq_issued;
            mbar_expect_tx(bar_tma, 2 * 16384);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_4d(sbase + P_IN + hf * 16384, &tm_k, hf * 64, ih, ic * C, ib, bar_tma);
                tma_load_4d(sbase + P_IN + hf * 16384 + 8192, &tm_q, hf * 64, ih, ic * C, ib, bar_tma);
            }
        };
        // Per-channel g: item j + 1's arrives by TMA while item j's operands
        // are built, and is scanned while item j's X product runs.
        auto issue_g = [&](int j) {
            int ib, ih, ic;
            item(j, ib, ih, ic);
            mbar_expect_tx(bar_g, 32768);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tma_load_4d(sbase + P_G + i * 8192, &tm_g, 32 * i, ih, ic * C, ib, bar_g);
        };
        auto beta_load = [&](int j, float (&bg)[4]) {
            int ib, ih, ic;
            item(j, ib, ih, ic);
            gate_scalar_load(ib, ih, ic, true, bg);
        };
        // Pool form: the record of the last item stored, published (its flag
        // set) once its stores are complete.
        unsigned int* pending_flag = nullptr;
        unsigned int pending_value = 0;
        long long pending_task = -1;
        auto publish = [&]() {
            bulk_wait_all();
            fence_proxy_async_global();
            if (pending_task != p.withheld_task) flag_release(pending_flag, pending_value);
            pending_flag = nullptr;
        };
        int g_issued = 0, g_waited = 0;          // g loads issued / waited for
        // Wait for a g tile, scan it in place (thread c < 128 runs the 64
        // tokens of channel c in order; a row of a box is 32 channels on 32
        // banks), then read this thread's values.  Every thread calls it.
        auto scan_g = [&](float (&gn)[4][8], int nvalid) {
            ok = ok && mbar_wait(bar_g, g_waited & 1, &g_pair_status_word);
            ++g_waited;
            if (PRO) {   // raw g: g = -min(softplus, 5) on the chunk's tokens, padding 0; all threads
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int f = tid + NT * j, r = f >> 5, c4 = f & 31;
                    float4* a = reinterpret_cast<float4*>(smem + P_G + (c4 >> 3) * 8192 + swz(r, c4 & 7));
                    float4 v = *a;
                    if (r < nvalid) {
                        const float2 lo = prologue_math::gate_fn2(make_float2(v.x, v.y));
                        const float2 hi = prologue_math::gate_fn2(make_float2(v.z, v.w));
                        v = make_float4(lo.x, lo.y, hi.x, hi.y);
                    } else {
                        v = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    *a = v;
                }
                __syncthreads();
            }
            if (tid < D) {
                uint8_t* col = smem + P_G + (tid >> 5) * 8192 + (tid & 3) * 4;
                const uint32_t cchunk = (tid & 31) >> 2;
                float acc = 0.f;
#pragma unroll
                for (int t0 = 0; t0 < C; t0 += 16) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = *reinterpret_cast<const float*>(col + swz(t0 + i, cchunk));
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        acc += v[i];
                        v[i] = acc;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) *reinterpret_cast<float*>(col + swz(t0 + i, cchunk)) = v[i];
                    if (t0 == 0) sRef0[tid] = v[15];          // token 15
                    if (t0 == 32) sRef1[tid] = v[15];         // token 47
                    if (POOL && t0 == 48) sLastP[tid] = v[15];   // token 63
                }
            }
            __syncthreads();
            const uint8_t* box = smem + P_G + (ck >> 2) * 8192;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = tg + 16 * u;
                const float4 a = *reinterpret_cast<const float4*>(box + swz(r, 2 * (ck & 3)));
                const float4 c = *reinterpret_cast<const float4*>(box + swz(r, 2 * (ck & 3) + 1));
                gn[u][0] = a.x; gn[u][1] = a.y; gn[u][2] = a.z; gn[u][3] = a.w;
                gn[u][4] = c.x; gn[u][5] = c.y; gn[u][6] = c.z; gn[u][7] = c.w;
            }
        };
        if (tid == 0 && nitems > 0) issue_kq(0);
        int kq_waited = -1;
        bool copy_pending = false;
        float gnext[4][8], bgnext[4];
        if (CHANNEL && nitems > 0) {
            if (tid == 0) { issue_g(0); g_issued = 1; }
            scan_g(gnext, item_valid(0));
            __syncthreads();                      // item 0's g has been read
            if (tid == 0 && nitems > 1) { issue_g(1); g_issued = 2; }
        }
        if (nitems > 0) {
            beta_load(0, bgnext);
            pro_load(0);
        }

        bool next_slot_free = false;           // tid 0: the next item's slot found free
        for (int ci = 0; ci < nitems; ++ci) {
            const bool slot_free = next_slot_free;
            next_slot_free = false;
            uint8_t* gslot = nullptr;           // pool form: this item's record slot
            int item_pair = 0, item_chunk = 0;
            if (POOL) {
                int ib, ih, ic;
                item(ci, ib, ih, ic);
                item_pair = ib * H + ih;
                item_chunk = ic;
                gslot = p.slots + ((size_t)item_pair * p.ring + ic % p.ring) * TASK_BYTES;
            }
            float gam[4][8];
            float2 last2[4];                    // pool form: G of the last token, this thread's channels
            float my_last = 0.f;                // pool form: G of the last token, channel tid
            if (CHANNEL) {   // scanned one chunk ahead; sRef0/1 hold this chunk's
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < 8; ++e) gam[u][e] = gnext[u][e];
            }
            // beta (and a scalar g) were loaded one chunk ahead.
            gate_scalar(bgnext, sGam, sBeta, sEr, sFj, sSafe);
            if (CHANNEL && ci + 1 < nitems) beta_load(ci + 1, bgnext);
            // (the fused prologue's next history rows and taps are loaded after
            // this item's conversion, below)
            ok = ok && mbar_wait(bar_tma, ci & 1, &g_pair_status_word);
            if (ok) kq_waited = ci;   // else drained at exit
            if (POOL && tid == 0 && item_chunk >= p.ring && !slot_free) {
                // The slot's previous record (chunk - ring) must have been
                // read by its chain before anything is stored into it
                // (usually found so already while the previous item's X ran).
                // The previous item's record is published first: a prep CTA
                // never waits while it holds a finished record, so that the
                // unfinished task of lowest index always has every earlier
                // record published (the ring's progress argument).
                if (copy_pending) {
                    publish();
                    copy_pending = false;
                }
                ok = ok && flag_wait_until(p.consumed + item_pair, (unsigned)(item_chunk - p.ring + 1),
                                           &g_pair_status_word);
                fence_proxy_async_global();
            }
            if (__syncthreads_or(!ok)) break;

            if constexpr (PRO) {
                // Fused prologue: the raw q and k tiles become the recurrence's
                // inputs in place, as gdn_prologue computes them (see
                // pro_convert_tile); the history rows and taps were loaded a
                // task ahead.
                float* sH = reinterpret_cast<float*>(smem + P_PH);
                float4* sW = reinterpret_cast<float4*>(smem + P_PW);
                float* sS = reinterpret_cast<float*>(smem + P_PS);
                {
                    const int tn = tid >> 7, ch = tid & 127;
#pragma unroll
                    for (int i = 0; i < 3; ++i) sH[(tn * 3 + i) * D + ch] = hq[i];
                    sW[tid] = tq;
                }
                __syncthreads();
                const int nvalid = T - item_chunk * C < C ? T - item_chunk * C : C;
                pro_convert_tile(smem + P_IN + 8192, 16384, sH, sW, sS, nvalid, p.silu, true, false, tid);
                pro_convert_tile(smem + P_IN, 16384, sH + 3 * D, sW + D, sS, nvalid, p.silu, true, false, tid);
            }

            if (CHANNEL) {
                // Channel pairs on the paired fp32 instructions.  Tokens
                // tg + 16u with u < 2 are before token 32 (reference 15).
                const float2 l2e = make_float2(kLog2e, kLog2e);
                float2 ref0[4], ref1[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ref0[e] = make_float2(sRef0[8 * ck + 2 * e], sRef0[8 * ck + 2 * e + 1]);
                    ref1[e] = make_float2(sRef1[8 * ck + 2 * e], sRef1[8 * ck + 2 * e + 1]);
                    if (POOL) last2[e] = make_float2(sLastP[8 * ck + 2 * e], sLastP[8 * ck + 2 * e + 1]);
                }
                if (POOL) my_last = tid < D ? sLastP[tid] : 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = tg + 16 * u;
                    float kf[8], qf[8];
                    load_bf16x8(smem + P_IN + ckh * 16384 + swz(r, ckc), kf);
                    load_bf16x8(smem + P_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
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
                    store_split2(smem + P_AH + o128, smem + P_AL + o128, kr);
                    store_split2(smem + P_AH + o128q, smem + P_AL + o128q, qr);
                    if (u < 2) {
                        const uint32_t o32 = ckh * 2 * CB_HALF + swz(r, ckc);
                        store_split2(smem + P_CB + o32, smem + P_CB + CB_HALF + o32, kc);
                    }
                    const uint32_t o64 = ckh * 2 * CB_HALF + swz(32 + r, ckc);
                    store_split2(smem + P_CB + o64, smem + P_CB + CB_HALF + o64, kc1);
                }
                fence_async_smem();
                __syncthreads();
            }
            if (tid == 0) {
                tc_fence_after();
                if (CHANNEL) {
                    // A hi times [B hi; B lo] (N = 192) into TM_X .. + 191, A lo
                    // times B hi into the first 96 columns; the epilogue adds
                    // the two 96-column halves.
                    const uint32_t id2 = idesc_bf16(128, 192, false, false);
                    const uint32_t id = idesc_bf16(128, 96, false, false);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t ka = (ks >> 2) * 16384 + (ks & 3) * 32;
                        const uint32_t kb = (ks >> 2) * 2 * CB_HALF + (ks & 3) * 32;
                        const uint64_t ah = sdesc_sw128(sbase + P_AH + ka, 16, 1024);
                        const uint64_t al = sdesc_sw128(sbase + P_AL + ka, 16, 1024);
                        const uint64_t bh = sdesc_sw128(sbase + P_CB + kb, 16, 1024);
                        mma_bf16(tmem + TM_X, ah, bh, id2, ks > 0);
                        mma_bf16(tmem + TM_X, al, bh, id, 1);
                    }
                } else {
                    const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint64_t a = sdesc_sw128(sbase + P_IN + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                        mma_bf16(tmem + TM_X, a, a, id, ks > 0);
                    }
                }
                mma_commit(sbase + P_BAR + 8);
                // Pool form: the previous item's record, whose stores have long
                // completed, is published here, before this thread issues new
                // global stores (a release waits for the thread's own stores).
                if (POOL && copy_pending) {
                    publish();
                    copy_pending = false;
                }
                // Pool form: the next item's record slot, tried while X runs
                // (the acquire's cost is hidden there).
                if (POOL && ci + 1 < nitems) {
                    int nb, nh, nc;
                    item(ci + 1, nb, nh, nc);
                    next_slot_free = nc < p.ring ||
                        (int)(flag_acquire(p.consumed + nb * H + nh) - (unsigned)(nc - p.ring + 1)) >= 0;
                }
            }
            // Fused prologue: the next task's history rows and taps, loaded
            // here, where no proxy fence follows soon (a shared-memory proxy
            // fence waits for the thread's own outstanding global loads).
            if (PRO && ci + 1 < nitems) pro_load(ci + 1);
            // While X runs: the chain's operands (pool form) and the next
            // chunk's g (the X build of this chunk has read sRef0/1 already).
            if (POOL && CHANNEL) {    // the chain's operands K*E, Q*E and K*D, exp(G_last)
                const float2 l2e = make_float2(kLog2e, kLog2e);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = tg + 16 * u;
                    float kf[8], qf[8], ke[8], qe[8];
                    float2 kd[4];
                    load_bf16x8(smem + P_IN + ckh * 16384 + swz(r, ckc), kf);
                    load_bf16x8(smem + P_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 k2 = make_float2(kf[2 * e], kf[2 * e + 1]);
                        const float2 q2 = make_float2(qf[2 * e], qf[2 * e + 1]);
                        const float2 g2 = make_float2(gam[u][2 * e], gam[u][2 * e + 1]);
                        const float2 el = mul2(g2, l2e);
                        const float2 dl = mul2(sub2(last2[e], g2), l2e);
                        const float2 E2 = make_float2(ex2_approx(el.x), ex2_approx(el.y));
                        const float2 D2 = make_float2(ex2_approx(dl.x), ex2_approx(dl.y));
                        const float2 ke2 = mul2(k2, E2), qe2 = mul2(q2, E2);
                        ke[2 * e] = ke2.x; ke[2 * e + 1] = ke2.y;
                        qe[2 * e] = qe2.x; qe[2 * e + 1] = qe2.y;
                        kd[e] = mul2(k2, D2);
                    }
                    const uint32_t oc = ckh * 8192 + swz(r, ckc);
                    store_bf16x8(gslot + TA_KE + oc, ke);
                    store_f16x8(gslot + TB_QE + oc, qe);
                    store_split2(gslot + TC_KD + oc, gslot + TC_KD + 16384 + oc, kd);
                }
                if (tid < D) reinterpret_cast<float*>(gslot + TC_EL)[tid] = __expf(my_last);
            }
            if (CHANNEL && ci + 1 < nitems) scan_g(gnext, item_valid(ci + 1));
            if (POOL && !CHANNEL) {   // the chain's operands Q*E and K*D, exp(G_last); K*E here
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = tg + 16 * u;
                    float kf[8], qf[8], ke[8], qe[8], kd[8];
                    load_bf16x8(smem + P_IN + ckh * 16384 + swz(r, ckc), kf);
                    load_bf16x8(smem + P_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
                    const float E = ex2_approx(sGam[r] * kLog2e);
                    const float Dd = ex2_approx((sGam[C - 1] - sGam[r]) * kLog2e);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        ke[e] = kf[e] * E;
                        qe[e] = qf[e] * E;
                        kd[e] = kf[e] * Dd;
                    }
                    const uint32_t oc = ckh * 8192 + swz(r, ckc);
                    store_bf16x8(smem + P_KE + oc, ke);     // for this CTA's W^T product
                    store_f16x8(gslot + TB_QE + oc, qe);
                    store_split(gslot + TC_KD + oc, gslot + TC_KD + 16384 + oc, kd);
                }
                if (tid < D) reinterpret_cast<float*>(gslot + TC_EL)[tid] = __expf(sGam[C - 1]);
            }
            mma_sync();
            if (!POOL && tid == 0 && copy_pending) {      // the staging is free again
                bulk_wait_read_all();
                copy_pending = false;
            }
            if (__syncthreads_or(!ok)) break;
            // Raw K, Q and the X operands are consumed: prefetch the next item;
            // the g tile has been read by every thread.
            if (tid == 0 && ci + 1 < nitems) issue_kq(ci + 1);
            if (CHANNEL && tid == 0 && ci + 2 < nitems) { issue_g(ci + 2); g_issued = ci + 3; }
            if (!CHANNEL && ci + 1 < nitems) beta_load(ci + 1, bgnext);

            // A and P from X (see chunk_sm100.cu); P as bf16 hi + lo into the staging.
            {
                const int L = quad * 32 + lane;
                const bool is_p = L >= 64;
                const int r = L & 63;
                float x[32];
                const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
                bool zero = false;
                if (CHANNEL) {
                    float x2[32];
                    const uint32_t col = r < 32 ? 0u : 32u + half * 32u;
                    zero = r < 32 && half != 0;
                    if (!zero) {
                        tmem_ld32(lane_base + TM_X + col, x);
                        tmem_ld32(lane_base + TM_X + 96 + col, x2);
                    }
                    tmem_wait_ld();
                    if (!zero) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) x[jj] += x2[jj];
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
                        store_split(smem + P_STAGE + 16384 + swz(r, cc), smem + P_STAGE + 24576 + swz(r, cc), pv);
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
            solve_unit_lower64_rd(sA, sT, sY, tid);
            if (POOL && CHANNEL) {   // T and beta as they are; the chain forms T'
                const float4* src = reinterpret_cast<const float4*>(sT);
                float4* dst = reinterpret_cast<float4*>(smem + P_STAGE);
                for (int e = tid; e < 1024; e += NT) dst[e] = src[e];
                if (tid < C) reinterpret_cast<float*>(gslot + TA_BETA)[tid] = sBeta[tid];
            }
            for (int e = tid; !(POOL && CHANNEL) && e < 512; e += NT) {
                const int r = e >> 3, c = e & 7;
                const float4 t0v = *reinterpret_cast<const float4*>(&sT[tidx(r, 8 * c)]);
                const float4 t1v = *reinterpret_cast<const float4*>(&sT[tidx(r, 8 * c + 4)]);
                const float tt[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
                float tv[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int m = 8 * c + q;
                    tv[q] = (m <= r) ? tt[q] * sBeta[m] : 0.f;
                }
                store_split(smem + P_STAGE + swz(r, c), smem + P_STAGE + 8192 + swz(r, c), tv);
            }
            fence_async_smem();          // staging written by threads -> read by the bulk copy
            __syncthreads();
            if (POOL && !CHANNEL) {
                // Scalar gate: W^T = (K*E)^T T'^T here, so that the chain,
                // the bound with a scalar gate, receives W ready-made (fp16,
                // the image of its operand tile) and runs one product round
                // trip less per chunk.
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t bt = sdesc_sw128(sbase + P_STAGE + part * 8192 + ks * 32, 16, 1024);
                            mma_bf16(tmem + TM_X, sdesc_sw128(sbase + P_KE + ks * 2048, 8192, 1024), bt, id,
                                     (part | ks) != 0);
                        }
                    }
                    mma_commit(sbase + P_BAR + 8);
                }
                mma_sync();
                float w[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_X + half * 32, w);
                tmem_wait_ld();
                const int wrow = quad * 32 + lane;
#pragma unroll
                for (int c = 0; c < 4; ++c) store_f16x8(gslot + TA_KE + swz(wrow, half * 4 + c), &w[8 * c]);
                tc_fence_before();
            }
            if (tid == 0 && !POOL) {
                // Wait until CTA 1 has consumed the previous chunk's slot.
                ok = ok && mbar_wait_cluster(bar_empty, (ci & 1) ^ 1, &g_pair_status_word);
                if (ok) {
                    mbar_arrive_expect_tx_remote_relaxed(peer_full, SLOT_BYTES);
                    bulk_copy_to_peer(peer_slot, sbase + P_STAGE, SLOT_BYTES, peer_full);
                    bulk_commit();
                    copy_pending = true;
                }
            }
            if (tid == 0 && POOL) {
                // T' and P to the task's record in the global buffer (its
                // other tiles were stored by every thread before the barrier
                // above); the flag is set once the stores are complete (at
                // once for the first item, which the chains wait for;
                // otherwise once the next item's X product is issued, when
                // the stores have long finished).
                bulk_store_global(gslot + TA_T, sbase + P_STAGE, 16384);            // T' or T
                bulk_store_global(gslot + TC_P, sbase + P_STAGE + 16384, 16384);    // P
                bulk_commit();
                pending_flag = p.flags + (size_t)item_pair * p.ring + item_chunk % p.ring;
                pending_value = (unsigned)item_chunk + 1u;
                pending_task = (long long)item_pair * nchunks + item_chunk;
                copy_pending = true;
                if (ci == 0) {
                    publish();
                    copy_pending = false;
                }
            }
            if (__syncthreads_or(!ok)) break;
        }
        if (tid == 0) {
            bulk_wait_all();                 // own copies complete before exit
            if (POOL && pending_flag) publish();
            for (int i = kq_waited + 1; !ok && i < kq_issued; ++i)   // K/Q tiles still in flight
                mbar_wait(bar_tma, i & 1, &g_pair_status_word);
            for (int i = g_waited; !ok && i < g_issued; ++i)   // g tiles still in flight
                mbar_wait(bar_g, i & 1, &g_pair_status_word);
        }
    } else {
        // ========================================================== chain CTA ===
        float* sGam = reinterpret_cast<float*>(smem + C_GAM);
        float* sLast = reinterpret_cast<float*>(smem + C_LAST);
        const uint32_t bar_kq = sbase + C_BAR, bar_v = sbase + C_BAR + 8;
        const uint32_t bar_full = sbase + C_BAR + 24;
        const uint32_t bar_mma = sbase + C_BAR + 16;
        // Products into O^T are committed apart (bar_out), so that the U
        // epilogue and the state update do not wait for them.
        const uint32_t bar_out = sbase + C_BAR + 32;
        const uint32_t peer_empty = POOL ? 0u : mapa_shared(sbase + P_BAR + 16, 0);
        // Pool form: chunk c's record is fetched from the global buffer in
        // three parts, each onto its own mbarrier, as soon as chunk c - 1's
        // products that read the same tiles are complete: part A (T', K*E)
        // after the W and U~ products, part B (Q*E) after the SN products (the
        // O products that read Q*E precede them), part C (P, K*D, exp(G_last))
        // once the chunk's output is staged.  The record's flag is tried early
        // in chunk c - 1 by the fetching thread, without blocking; when set,
        // the record is also prefetched into L2 (prep CTAs may run far ahead
        // of the chains, and records written long before have left L2).  The
        // counts of parts fetched are kept in shared memory for the drain on
        // an abandoned wait.  The chain then needs no raw K, Q or gate, and W^T
        // goes to the raw K, Q tile instead of over K*E.
        const uint32_t bar_full_b = sbase + C_BAR + 40, bar_full_c = sbase + C_BAR + 48;
        const uint32_t C_W = POOL ? C_IN : C_KE;
        // Pool form, scalar gate: W^T arrives in the record (part A, over the
        // K*E tile) and the chain skips its own W^T product.
        constexpr bool W_READY = POOL && !CHANNEL;
        const uint32_t C_WB = W_READY ? C_KE : C_W;
        const uint32_t C_TF = C_IN + 16384;    // pool form, per-channel: T fp32 (tidx layout)
        int* sFetched = reinterpret_cast<int*>(smem + C_FETCHED);
        int acquired = -1;              // chunk whose flag this thread has acquired
        auto record = [&](int chunk) {
            return p.slots + ((size_t)pair * p.ring + chunk % p.ring) * TASK_BYTES;
        };
        auto flag_of = [&](int chunk) { return p.flags + (size_t)pair * p.ring + chunk % p.ring; };
        auto try_acquire = [&](int chunk) {
            if (flag_acquire(flag_of(chunk)) != (unsigned)chunk + 1u) return;
            fence_proxy_async_global();
            bulk_prefetch_l2(record(chunk), TASK_BYTES);
            acquired = chunk;
        };
        auto fetch_part = [&](int chunk, int part) {
            if (acquired != chunk) {
                ok = ok && flag_wait_until(flag_of(chunk), (unsigned)chunk + 1u, &g_pair_status_word,
                                           p.flag_budget_ns);
                if (!ok) return;
                fence_proxy_async_global();
                acquired = chunk;
            }
            const uint8_t* rec = record(chunk);
            if (part == 0) {
                mbar_expect_tx(bar_full, CHANNEL ? PART_A + 256 : PART_A);
                bulk_load_global(sbase + (CHANNEL ? C_TF : C_TH), rec + TA_T, 16384, bar_full);
                bulk_load_global(sbase + C_KE, rec + TA_KE, 16384, bar_full);
                if (CHANNEL) bulk_load_global(sbase + C_GAM, rec + TA_BETA, 256, bar_full);
            } else if (part == 1) {
                mbar_expect_tx(bar_full_b, PART_B);
                bulk_load_global(sbase + C_QE, rec + TB_QE, 16384, bar_full_b);
            } else {
                mbar_expect_tx(bar_full_c, PART_C);
                bulk_load_global(sbase + C_PH, rec + TC_P, 16384, bar_full_c);
                bulk_load_global(sbase + C_KDH, rec + TC_KD, 32768, bar_full_c);
                bulk_load_global(sbase + C_LAST, rec + TC_EL, 512, bar_full_c);
            }
            sFetched[part] = chunk + 1;
        };
        if (POOL && tid == 0) sFetched[0] = sFetched[1] = sFetched[2] = 0;
        auto discard_record = [&](int chunk) {
            const uint8_t* rec = record(chunk);
            for (uint32_t off = tid * 128u; off < TASK_BYTES; off += NT * 128u) discard_l2_line(rec + off);
        };

        const int srow = quad * 32 + lane;
        const int scol = half * 64;
        float s[64];
        const long DD = (long)D * D;
        if (p.state_in) {
            const float4* src = reinterpret_cast<const float4*>(p.state_in + ((long)b * H + h) * DD +
                                                                (long)srow * D + scol);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float4 t = src[c];
                s[4 * c] = t.x; s[4 * c + 1] = t.y; s[4 * c + 2] = t.z; s[4 * c + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = 0.f;
        }
        auto write_state_f16 = [&]() {
            uint8_t* dst = smem + C_S + half * 16384;
#pragma unroll
            for (int c = 0; c < 8; ++c) store_f16x8(dst + swz(srow, c), &s[8 * c]);
        };
        write_state_f16();
        int kq_issued = 0, v_issued = 0;   // loads issued (tid 0), for the drain
        auto issue_kq = [&](int chunk) {
            const int t0 = chunk * C;
            ++kq_issued;
            mbar_expect_tx(bar_kq, 2 * 16384);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_4d(sbase + C_IN + hf * 16384, &tm_k, hf * 64, h, t0, b, bar_kq);
                tma_load_4d(sbase + C_IN + hf * 16384 + 8192, &tm_q, hf * 64, h, t0, b, bar_kq);
            }
        };
        auto issue_v = [&](int chunk) {
            const int t0 = chunk * C;
            ++v_issued;
            mbar_expect_tx(bar_v, 16384);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                tma_load_4d(sbase + C_V + hf * 8192, &tm_v, hf * 64, h, t0, b, bar_v);
        };
        fence_async_smem();
        __syncthreads();
        if (tid == 0 && nchunks > 0) {
            if (!POOL) issue_kq(0);
            issue_v(0);
        }
        int kq_waited = -1, v_waited = -1, full_waited = -1, b_waited = -1, c_waited = -1;
        float gnext[4][8], bgnext[4];
        if (!POOL && CHANNEL && nchunks > 0) gate_load(0, gnext);
        if (!POOL && !CHANNEL && nchunks > 0) gate_scalar_load(b, h, 0, false, bgnext);
        // Per-channel: chunk 0's scan here; the scan of chunk c + 1 runs
        // while the products SN of chunk c are on the tensor core.
        if (!POOL && CHANNEL && nchunks > 0) gate_channel(0, (long)b * T * H + h, gnext, nullptr, nullptr, sLast);
        if (POOL && tid == 0 && nchunks > 0) {
            fetch_part(0, 0);
            fetch_part(0, 1);
            fetch_part(0, 2);
        }
        // Fused prologue: v's taps (conv channels 2D .. 3D - 1 of this head)
        // and chunk 0's history rows of v (tokens -3 .. -1: the ring or zero;
        // thread tid < 128 takes channel tid) once; each later chunk's history
        // is its predecessor's raw last three tokens, kept by the conversion.
        float hv[3] = {0.f, 0.f, 0.f};
        auto pro_load_v = [&](int chunk) {
            if (!PRO || tid >= D) return;
            const int p0 = p.pos0 ? p.pos0[b] : 0;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const int t = chunk * C - 3 + i;
                float x = 0.f;
                if (t >= 0) x = __bfloat162float(p.v_raw[(((long)b * T + t) * H + h) * D + tid]);
                else if (p.conv_ring && p0 + t >= 0)
                    x = p.conv_ring[(((long)b * H + h) * 4 + ((p0 + t) & 3)) * (3 * D) + 2 * D + tid];
                hv[i] = x;
            }
        };
        auto pro_store_v = [&]() {
            if (!PRO || tid >= D) return;
            float* sHV = reinterpret_cast<float*>(smem + C_HV);
#pragma unroll
            for (int i = 0; i < 3; ++i) sHV[i * D + tid] = hv[i];
        };
        if (PRO) {
            if (tid < D)
                reinterpret_cast<float4*>(smem + C_TV)[tid] =
                    *reinterpret_cast<const float4*>(p.conv_w + ((long)h * 3 * D + 2 * D + tid) * 4);
            if (nchunks > 0) {       // chunk 0's history; later chunks keep their predecessor's
                pro_load_v(0);
                pro_store_v();
            }
        }
        // A first record that never came: no chunk starts (every thread
        // learns it here, before any wait of the loop).
        const bool started = !POOL || !__syncthreads_or(!ok);

        for (int ci = 0; started && ci < nchunks; ++ci) {
            const int t0 = ci * C;
            const long tk0 = ((long)b * T + t0) * H + h;
            float e_last = 0.f;
          if (!POOL) {   // the operands K*E, Q*E, K*D from raw K, Q and the gate
            float gam[4][8];
            if (CHANNEL) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int e = 0; e < 8; ++e) gam[u][e] = gnext[u][e];   // already scanned
            } else {
                gate_scalar(bgnext, sGam, nullptr);
            }
            ok = ok && mbar_wait(bar_kq, ci & 1, &g_pair_status_word);
            if (ok) kq_waited = ci;   // else drained at exit
            if (__syncthreads_or(!ok)) break;

            // K*E (bf16), Q*E (fp16), K*D (bf16 hi + lo), on channel pairs.
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
                    load_bf16x8(smem + C_IN + ckh * 16384 + swz(r, ckc), kf);
                    load_bf16x8(smem + C_IN + ckh * 16384 + 8192 + swz(r, ckc), qf);
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
                    store_bf16x8(smem + C_KE + o64, ke);
                    store_f16x8(smem + C_QE + o64, qe);
                    store_split2(smem + C_KDH + o64, smem + C_KDL + o64, kd);
                }
            }
            e_last = __expf(CHANNEL ? sLast[srow] : sGam[C - 1]);
            fence_async_smem();
            __syncthreads();
            if (tid == 0 && ci + 1 < nchunks) issue_kq(ci + 1);   // raw K, Q consumed
            if (ci + 1 < nchunks) {
                if (CHANNEL) gate_load(ci + 1, gnext);
                else gate_scalar_load(b, h, ci + 1, false, bgnext);
            }
          }

            // T' (with P, or pool form: with K*E) of this chunk from the prep
            // side; V of this chunk.
            if (tid == 0 || (POOL && CHANNEL)) {   // pool, per-channel: every thread reads T
                ok = ok && (POOL ? mbar_wait(bar_full, ci & 1, &g_pair_status_word)
                                 : mbar_wait_cluster(bar_full, ci & 1, &g_pair_status_word));
                if (ok) full_waited = ci;   // else drained at exit
            }
            if (POOL && CHANNEL && ok) {   // T' = T Diag(beta) as bf16 hi + lo (lower triangle)
                const float* sTc = reinterpret_cast<const float*>(smem + C_TF);
                const float* sBc = reinterpret_cast<const float*>(smem + C_GAM);
                for (int e = tid; e < 512; e += NT) {
                    const int r = e >> 3, c = e & 7;
                    const float4 t0v = *reinterpret_cast<const float4*>(&sTc[tidx(r, 8 * c)]);
                    const float4 t1v = *reinterpret_cast<const float4*>(&sTc[tidx(r, 8 * c + 4)]);
                    const float tt[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
                    float tv[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int m = 8 * c + q;
                        tv[q] = (m <= r) ? tt[q] * sBc[m] : 0.f;
                    }
                    store_split(smem + C_TH + swz(r, c), smem + C_TL + swz(r, c), tv);
                }
                fence_async_smem();
            }
            ok = ok && mbar_wait(bar_v, ci & 1, &g_pair_status_word);
            if (ok) v_waited = ci;   // else drained at exit
            if (__syncthreads_or(!ok)) break;
            if constexpr (PRO) {
                // Fused prologue: the raw v tile becomes the recurrence's v in
                // place (convolution, activation, bf16; no norm).
                pro_convert_tile(smem + C_V, 8192, reinterpret_cast<float*>(smem + C_HV),
                                 reinterpret_cast<const float4*>(smem + C_TV), nullptr,
                                 T - t0 < C ? T - t0 : C, p.silu, false, true, tid);
            }

          if (!W_READY) {
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint32_t tb = part ? C_TL : C_TH;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t bt = sdesc_sw128(sbase + tb + ks * 32, 16, 1024);
                        const uint32_t acc = (part | ks) != 0;
                        mma_bf16(tmem + TM_WT, sdesc_sw128(sbase + C_KE + ks * 2048, 8192, 1024), bt, id, acc);
                        mma_bf16(tmem + TM_UT, sdesc_sw128(sbase + C_V + ks * 2048, 8192, 1024), bt, id, acc);
                    }
                }
                mma_commit(bar_mma);
            }
            // Pool form: the next chunk's flag, tried while these products run.
            if (POOL && tid == NT - 32 && ci + 1 < nchunks) try_acquire(ci + 1);
            mma_sync();
            if (__syncthreads_or(!ok)) break;
            if (tid == 0 && ci + 1 < nchunks) issue_v(ci + 1);      // V consumed
            if (POOL && tid == NT - 32 && ci + 1 < nchunks) fetch_part(ci + 1, 0);   // T', K*E consumed

            {   // W^T -> fp16 [128 i][64 r] (over the consumed K*E tile, or pool form: raw K, Q's)
                float w[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_WT + half * 32, w);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) store_f16x8(smem + C_W + swz(srow, half * 4 + c), &w[8 * c]);
            }
          }
            if (POOL && !W_READY && tid == 0) {   // Q*E of this chunk, for the O products below
                ok = ok && mbar_wait(bar_full_b, ci & 1, &g_pair_status_word);
                if (ok) b_waited = ci;   // else drained at exit
            }
            fence_async_smem();
            tc_fence_before();
            if (!W_READY && __syncthreads_or(!ok)) break;
            // Pool form with W^T in the record: the next chunk's flag, tried
            // while the products below run.
            if (W_READY && tid == NT - 32 && ci + 1 < nchunks) try_acquire(ci + 1);

            if (tid == 0) {
                tc_fence_after();
                const uint32_t id_u = idesc_f16(128, 64, true, true, true);
                const uint32_t id_o = idesc_f16(128, 64, true, false);
                if (W_READY) {   // U~^T = V^T T'^T first (W^T came with the record)
                    const uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        const uint32_t tb = part ? C_TL : C_TH;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + TM_UT, sdesc_sw128(sbase + C_V + ks * 2048, 8192, 1024),
                                     sdesc_sw128(sbase + tb + ks * 32, 16, 1024), id, (part | ks) != 0);
                    }
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = sdesc_sw128(sbase + C_S + ks * 2048, 16384, 1024);
                    mma_bf16(tmem + TM_UT, a, sdesc_sw128(sbase + C_WB + ks * 2048, 8192, 1024), id_u, 1);
                }
                mma_commit(bar_mma);
                if (W_READY) {           // Q*E of this chunk, for the O products below
                    ok = ok && mbar_wait(bar_full_b, ci & 1, &g_pair_status_word);
                    if (ok) b_waited = ci;   // else drained at exit
                }
              if (ok) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = sdesc_sw128(sbase + C_S + ks * 2048, 16384, 1024);
                    const uint64_t bq = sdesc_sw128(sbase + C_QE + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                    mma_bf16(tmem + TM_OT, a, bq, id_o, ks > 0);
                }
              }
            }
            mma_sync();
            if (W_READY) {   // V, T' and W^T are consumed (the U~ and U products are complete)
                if (tid == 0 && ci + 1 < nchunks) issue_v(ci + 1);
                if (tid == NT - 32 && ci + 1 < nchunks) fetch_part(ci + 1, 0);
            }
            if (tid == 0) bulk_wait_read_all();   // the previous O store has read C_OST
            if (__syncthreads_or(!ok)) break;

            {   // U^T -> bf16 hi + lo [128 j][64 r]
                float u[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TM_UT + half * 32, u);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    store_split(smem + C_UH + swz(srow, half * 4 + c), smem + C_UL + swz(srow, half * 4 + c),
                                &u[8 * c]);
            }
            if (POOL && tid == 0) {          // P and K*D of this chunk, for the products below
                ok = ok && mbar_wait(bar_full_c, ci & 1, &g_pair_status_word);
                if (ok) c_waited = ci;   // else drained at exit
            }
            fence_async_smem();
            tc_fence_before();
            if (__syncthreads_or(!ok)) break;

            if (tid == 0) {
                tc_fence_after();
                const uint32_t id_s = idesc_bf16(128, 128, true, false);
                const uint32_t id_o = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t kdh = sdesc_sw128(sbase + C_KDH + ks * 2048, 8192, 1024);
                    const uint64_t kdl = sdesc_sw128(sbase + C_KDL + ks * 2048, 8192, 1024);
                    const uint64_t uh = sdesc_sw128(sbase + C_UH + ks * 32, 16, 1024);
                    const uint64_t ul = sdesc_sw128(sbase + C_UL + ks * 32, 16, 1024);
                    mma_bf16(tmem + TM_SN, kdh, uh, id_s, ks > 0);
                    mma_bf16(tmem + TM_SN, kdh, ul, id_s, 1);
                    mma_bf16(tmem + TM_SN, kdl, uh, id_s, 1);
                }
                mma_commit(bar_mma);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t uh = sdesc_sw128(sbase + C_UH + ks * 32, 16, 1024);
                    const uint64_t ul = sdesc_sw128(sbase + C_UL + ks * 32, 16, 1024);
                    const uint64_t ph = sdesc_sw128(sbase + C_PH + ks * 32, 16, 1024);
                    const uint64_t pl = sdesc_sw128(sbase + C_PL + ks * 32, 16, 1024);
                    mma_bf16(tmem + TM_OT, uh, ph, id_o, 1);
                    mma_bf16(tmem + TM_OT, uh, pl, id_o, 1);
                    mma_bf16(tmem + TM_OT, ul, ph, id_o, 1);
                }
                mma_commit(bar_out);
            }
            if (!POOL && CHANNEL && ci + 1 < nchunks)   // sLast of this chunk is no longer read
                gate_channel(t0 + C, tk0 + (long)C * H, gnext, nullptr, nullptr, sLast);
            // Pool form, while these products run: the previous chunk's record
            // has been read for the last time, so its lines leave L2 without
            // a write-back (three lines per thread).
            if (POOL && ci > 0) discard_record(ci - 1);
            // Records of chunks < ci - 1 are read and were discarded in the
            // previous chunk, before its barriers: their slots may be reused.
            // (Released here, where this thread waits for the products anyway:
            // the release's fence costs the chain nothing.)
            if (POOL && p.ring < nchunks && tid == 32 && ci > 1)
                flag_release(p.consumed + pair, (unsigned)(ci - 1));
            mma_sync();
            if (__syncthreads_or(!ok)) break;
            if (POOL && tid == NT - 32 && ci + 1 < nchunks) fetch_part(ci + 1, 1);   // Q*E consumed
            if (POOL) {   // exp(G_last) arrived with part C
                ok = ok && mbar_wait(bar_full_c, ci & 1, &g_pair_status_word);
                e_last = sLast[srow];
            }

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
                        float2 a = fma2(e2, make_float2(s[c], s[c + 1]), make_float2(sn0[c], sn0[c + 1]));
                        float2 z = fma2(e2, make_float2(s[32 + c], s[33 + c]), make_float2(sn1[c], sn1[c + 1]));
                        s[c] = a.x; s[c + 1] = a.y; s[32 + c] = z.x; s[33 + c] = z.y;
                    }
                }
                write_state_f16();
                // Products into O^T complete (they read P in the slot and U^T):
                // the slot is free.  Cluster form: it goes back to CTA 0 (the
                // arrive is made by a thread of the last warp, which has no
                // global loads in flight).
                ok = ok && mbar_wait(bar_out, ci & 1, &g_pair_status_word);
                if (!POOL && tid == NT - 32 && ok) mbar_arrive_remote_relaxed(peer_empty);
                tc_fence_after();
                float o[32];
                tmem_ld32(lb + TM_OT + half * 32, o);
                tmem_wait_ld();
                // O^T (lane = value column) -> [token][column] fp32; one TMA
                // store writes the chunk and drops rows past T.  Global stores
                // from the threads would hold up the proxy fence below.
                float* so = reinterpret_cast<float*>(smem + C_OST) + half * 32 * D + srow;
#pragma unroll
                for (int r = 0; r < 32; ++r) so[r * D] = o[r];
            }
            fence_async_smem();
            tc_fence_before();
            if (__syncthreads_or(!ok)) break;
            if (tid == 0) {
                tma_store_4d(&tm_o, sbase + C_OST, 0, h, t0, b);
                bulk_commit();
            }
            // Pool form: P, K*D and exp(G_last) are consumed (every thread has
            // read its decay before the barrier above).
            if (POOL && tid == NT - 32 && ci + 1 < nchunks) fetch_part(ci + 1, 2);
        }
        if (tid == 0) bulk_wait_all();       // output stores complete before exit
        const bool failed = __syncthreads_or(!ok);
        if (tid == 0 && failed) {   // drain this CTA's own loads and products (bounded)
            for (int i = kq_waited + 1; !POOL && i < kq_issued; ++i) mbar_wait(bar_kq, i & 1, &g_pair_status_word);
            for (int i = v_waited + 1; i < v_issued; ++i) mbar_wait(bar_v, i & 1, &g_pair_status_word);
            if (POOL) {   // record parts still in flight (at most one of each)
                const int waited[3] = {full_waited, b_waited, c_waited};
                const uint32_t bars[3] = {bar_full, bar_full_b, bar_full_c};
                for (int q = 0; q < 3; ++q)
                    for (int i = waited[q] + 1; i < sFetched[q]; ++i)
                        mbar_wait(bars[q], i & 1, &g_pair_status_word);
            }
            mma_commit(bar_mma);
            mbar_wait(bar_mma, mma_phase, &g_pair_status_word);
            // Nothing of this chain reads its records any more: prep CTAs
            // waiting for its slots go on (their records are never read).
            if (POOL) flag_release(p.consumed + pair, 0x7fffffffu);
        }
        if (POOL && !failed && nchunks > 0) discard_record(nchunks - 1);   // every product has completed
        if (!failed && p.state_out) {
            float4* dst = reinterpret_cast<float4*>(p.state_out + ((long)b * H + h) * DD +
                                                    (long)srow * D + scol);
#pragma unroll
            for (int c = 0; c < 16; ++c) dst[c] = make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        }
    }

    // Neither CTA of a cluster leaves while the other may still touch its
    // shared memory.
    tc_fence_before();
    __syncthreads();
    if (!POOL) cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

template <bool CHANNEL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
chunk_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ CUtensorMap tm_g, const PairParams p)
{
    pair_body<CHANNEL, false>(tm_q, tm_k, tm_v, tm_o, tm_g, p);
}

template <bool CHANNEL>
__global__ void __launch_bounds__(NT, 1)
chunk_pool_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ CUtensorMap tm_g, const PairParams p)
{
    pair_body<CHANNEL, true>(tm_q, tm_k, tm_v, tm_o, tm_g, p);
}

// The pool form with the layer's input prologue applied while loading.
template <bool CHANNEL>
__global__ void __launch_bounds__(NT, 1)
chunk_pool_prologue_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                           const __grid_constant__ CUtensorMap tm_g, const PairParams p)
{
    pair_body<CHANNEL, true, true>(tm_q, tm_k, tm_v, tm_o, tm_g, p);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // Same entry point for every device; initialised once, thread-safely.
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

// out [B, T, H, D] fp32, box = one chunk of one head, no swizzle.
bool make_out_map(CUtensorMap* map, void* base, int H, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4, (cuuint64_t)T * H * D * 4};
    cuuint32_t box[4] = {(cuuint32_t)D, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// g [B, T, H, D] fp32 (per-channel gate), box 32 channels x 64 tokens, 128B swizzle.
bool make_g_map(CUtensorMap* map, const float* base, int H, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4, (cuuint64_t)T * H * D * 4};
    cuuint32_t box[4] = {32, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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

// Pool-form launch shared by the plain and the fused-prologue kernels: the
// task-record ring from the stream-ordered workspace (flags and counters
// first, 1 KB aligned, cleared on the stream before the launch), then one
// cooperative launch of pool_ctas CTAs.  Ring depth: every chunk gets its own
// slot while all records fit in kPoolScratchBytes (no slot is reused, so
// nothing waits for a chain); beyond that, as many slots per (batch, head)
// as fit, at least kPoolRing.  *too_large: the cooperative launch could not
// fit (only the memset ran).
template <typename Kernel>
cudaError_t launch_pool_ring(Kernel kernel, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, const CUtensorMap& mo, const CUtensorMap& mg,
                             PairParams prm, int nbh, int nchunks, int pool_ctas, cudaStream_t stream,
                             bool* too_large) {
    *too_large = false;
    long ring_max = (long)(kPoolScratchBytes / ((size_t)nbh * TASK_BYTES));
    if (ring_max < kPoolRing) ring_max = kPoolRing;
    if (const char* r = getenv("GDN_TEST_POOL_RING")) {   // tuning hook: another ring depth (>= 4)
        const int v = atoi(r);
        if (v >= 4) ring_max = v;
    }
    const int ring = nchunks < ring_max ? nchunks : (int)ring_max;
    const size_t nslots = (size_t)nbh * ring;
    const size_t counter_words = nslots + (size_t)nbh;
    const size_t flag_bytes = (counter_words * sizeof(unsigned int) + 1023) / 1024 * 1024;
    uint8_t* ws = nullptr;
    cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&ws), flag_bytes + nslots * TASK_BYTES, stream);
    if (e != cudaSuccess) return e;
    prm.flags = reinterpret_cast<unsigned int*>(ws);
    prm.consumed = prm.flags + nslots;
    prm.ring = ring;
    prm.slots = ws + flag_bytes;
    e = cudaMemsetAsync(ws, 0, counter_words * sizeof(unsigned int), stream);
    if (e == cudaSuccess) {
        // Cooperative: every CTA is resident at once (the chains wait on prep
        // CTAs), or the launch fails instead of starting.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pool_ctas);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, mo, mg, prm);
        if (e == cudaErrorCooperativeLaunchTooLarge) {
            if (cudaPeekAtLastError() == cudaErrorCooperativeLaunchTooLarge) (void)cudaGetLastError();
            *too_large = true;
            e = cudaSuccess;
        }
    }
    const cudaError_t ef = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : ef;
}

// Failure-detection test hooks of the pool form's flag wait: a task whose
// record is never published, and a short budget for the chains' flag waits.
// Unset in normal use.
void apply_test_hooks(PairParams& prm) {
    if (const char* w = getenv("GDN_TEST_WITHHOLD_TASK")) prm.withheld_task = atoll(w);
    if (const char* b = getenv("GDN_TEST_FLAG_BUDGET_NS")) {
        const long long ns = atoll(b);
        if (ns > 0) prm.flag_budget_ns = (unsigned long long)ns;
    }
}

template <bool CHANNEL>
cudaError_t launch_pair(const Problem& p, cudaStream_t stream, int pool_ctas) {
    {
        cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(chunk_pair_kernel<CHANNEL>), SMEM_BYTES);
        if (e == cudaSuccess)
            e = set_smem_limit(reinterpret_cast<const void*>(chunk_pool_kernel<CHANNEL>), SMEM_BYTES);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mk, mv, mo, mg;
    if (!make_map(&mq, p.q, p.H, p.T, p.B) || !make_map(&mk, p.k, p.H, p.T, p.B) ||
        !make_map(&mv, p.v, p.H, p.T, p.B) || !make_out_map(&mo, p.out, p.H, p.T, p.B))
        return cudaErrorInvalidValue;
    if (CHANNEL) {
        if (!make_g_map(&mg, p.g, p.H, p.T, p.B)) return cudaErrorInvalidValue;
    } else {
        mg = mq;                                   // not read with a scalar gate
    }
    PairParams prm{p.g, p.beta, p.state_in, p.state_out, static_cast<float*>(p.out), p.T, p.H, p.B,
                   nullptr, nullptr, nullptr, 0, kWaitBudgetNs, -1};
    apply_test_hooks(prm);
    const int nbh = p.B * p.H;
    const int nchunks = (p.T + C - 1) / C;
    bool too_large = pool_ctas <= nbh || nchunks == 0;
    if (!too_large) {
        cudaError_t e = launch_pool_ring(chunk_pool_kernel<CHANNEL>, mq, mk, mv, mo, mg, prm, nbh, nchunks,
                                         pool_ctas, stream, &too_large);
        if (e != cudaSuccess || !too_large) return e;
    }
    // The cluster form: a cluster of two CTAs per pair (fewer SMs free, or
    // the cluster form asked for).
    chunk_pair_kernel<CHANNEL><<<2 * nbh, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mo, mg, prm);
    return cudaGetLastError();
}

template <bool CHANNEL>
cudaError_t launch_pool_pro(const ProPrefill& a, cudaStream_t stream, bool* too_large) {
    const PrologueArgs& r = a.pro;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(chunk_pool_prologue_kernel<CHANNEL>), SMEM_BYTES);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, mo, mg;
    if (!make_map(&mq, r.q_raw, r.H, r.T, r.B) || !make_map(&mk, r.k_raw, r.H, r.T, r.B) ||
        !make_map(&mv, r.v_raw, r.H, r.T, r.B) || !make_out_map(&mo, a.out, r.H, r.T, r.B))
        return cudaErrorInvalidValue;
    if (CHANNEL) {
        if (!make_g_map(&mg, r.g_raw, r.H, r.T, r.B)) return cudaErrorInvalidValue;
    } else {
        mg = mq;
    }
    PairParams prm{r.g_raw, r.beta_raw, a.state_in, a.state_out, a.out, r.T, r.H, r.B,
                   nullptr, nullptr, nullptr, 0, kWaitBudgetNs, -1};
    apply_test_hooks(prm);
    prm.conv_w = r.conv_w;
    prm.conv_ring = r.ring;
    prm.pos0 = r.pos0;
    prm.q_raw = r.q_raw;
    prm.k_raw = r.k_raw;
    prm.v_raw = r.v_raw;
    prm.silu = r.silu;
    const int nbh = r.B * r.H;
    return launch_pool_ring(chunk_pool_prologue_kernel<CHANNEL>, mq, mk, mv, mo, mg, prm, nbh,
                            (r.T + C - 1) / C, sm_count(), stream, too_large);
}

}  // namespace

cudaError_t launch_chunk_pair_sm100(const Problem& p, cudaStream_t stream, int pool_ctas) {
    if (p.io_f32 || !p.out_f32 || p.dk != D || p.dv != D) return cudaErrorNotSupported;
    return p.per_channel ? launch_pair<true>(p, stream, pool_ctas) : launch_pair<false>(p, stream, pool_ctas);
}

cudaError_t launch_chunk_pool_prologue(const ProPrefill& a, cudaStream_t stream) {
    const PrologueArgs& r = a.pro;
    if (r.dk != D || r.dv != D || r.T < 1 || 2 * r.B * r.H > sm_count()) return cudaErrorNotSupported;
    bool too_large = false;
    cudaError_t e = r.per_channel ? launch_pool_pro<true>(a, stream, &too_large)
                                  : launch_pool_pro<false>(a, stream, &too_large);
    if (e != cudaSuccess) return e;
    if (too_large) return cudaErrorNotSupported;   // fewer SMs free: the caller runs the two passes
    if (r.ring) e = launch_prologue_ring(r, stream);   // after the kernel that read it
    return e;
}

cudaError_t read_and_clear_pair_status(unsigned int* status) {
    cudaError_t e = cudaMemcpyFromSymbol(status, g_pair_status_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_pair_status_word, &zero, sizeof(unsigned int));
}

}  // namespace gdn
