// gdn_internal.cuh -- declarations shared by the CUDA sources of libgdn.
// Not part of the public ABI (that is include/gdn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Arguments of one recurrence call, already validated by the ABI layer.
// Token-major layouts: q, k [B, T, H, dk]; v, out [B, T, H, dv];
// g [B, T, H] or [B, T, H, dk]; beta [B, T, H]; states [B, H, dk, dv].
// A decode step is the T = 1 case of the same layout ([B, H, d]).
struct Problem {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* state_in;   // may be null (zero state)
    float* state_out;        // may be null (not written)
    void* out;
    int B, T, H, dk, dv;
    bool per_channel;
    bool io_f32;             // q, k, v in fp32 (else bf16)
    bool out_f32;            // out in fp32 (else bf16)
    int segments = 0;        // chunk path: time segments per (b, h); 0 = automatic
    float* snapshots = nullptr;   // token-serial path: S after every token, [B, T, H, dk, dv]
    const float* beta_write = nullptr;   // token-serial path: separate write gate, [B, T, H]
};

// Token-serial fused recurrence (decode, and the fp32 / fallback prefill).
cudaError_t launch_recurrent(const Problem& p, cudaStream_t stream);

// state_out[b] := snapshots[b, n_b - 1] for 1 <= n_b <= T (n = num_accepted,
// device memory); other rows are left as they are.
cudaError_t launch_state_select(const float* snapshots, const int* num_accepted, float* state_out,
                                int B, int T, int H, int dk, int dv, cudaStream_t stream);

// Gradients of the chunkwise recurrence (chunk_bwd.cu).  bf16 q, k, v; fp32
// everything else; gradients in fp32.
struct BwdProblem {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* g;
    const float* beta;
    const float* state_in;      // may be null (zero)
    const float* d_out;         // [B, T, H, dv]
    const float* d_state_out;   // [B, H, dk, dv] or null (zero)
    float* dq;
    float* dk;
    float* dv;
    float* dg;
    float* dbeta;
    float* d_state_in;          // may be null (not written)
    int B, T, H, Dk, Dv;
    bool per_channel;
};
cudaError_t launch_chunk_bwd(const BwdProblem& p, cudaStream_t stream);

// Stream-ordered scratch from the library's per-device memory pool (freed
// with cudaFreeAsync on the same stream).
cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to the device that is current when it is
// set, so it is set once per (device, kernel), under a lock.
cudaError_t set_smem_limit(const void* kernel, int bytes);

// Number of SMs of the current device (looked up once per device).
int sm_count();

// Chunkwise tensor-core prefill (bf16 I/O, dk = dv = 128, chunk of 64).
// Returns cudaErrorNotSupported for shapes it does not handle.
cudaError_t launch_chunk_sm100(const Problem& p, cudaStream_t stream);

// The segment-parallel chunk path with its scratch taken from a fixed
// device array of kNoAllocScratchFloats floats instead of an allocation.
// Sets *over_limit (and launches nothing) when the call needs more.
constexpr size_t kNoAllocScratchFloats = size_t(8) * 1024 * 1024;   // 32 MiB
cudaError_t launch_chunk_sm100_noalloc(const Problem& p, cudaStream_t stream, bool* over_limit);

// The same chunk algebra with the chunk-local work (A, P, T') and the state
// chain of each (batch, head) on different SMs.  pool_ctas <= B * H: a
// cluster of two CTAs per pair (one prepares chunk c + 1 while the other runs
// the chain of chunk c).  pool_ctas > B * H: one cooperative grid of that
// many CTAs, B * H chains and the rest prep CTAs that share every pair's
// chunks through a global buffer of task records.  Used for unsegmented calls when
// 2 * B * H <= #SMs.
cudaError_t launch_chunk_pair_sm100(const Problem& p, cudaStream_t stream, int pool_ctas);
cudaError_t read_and_clear_pair_status(unsigned int* status);

// The layer's input prologue (prologue.cu): width-4 causal convolution over
// q | k | v with a 4-slot history ring, SiLU or none, q/k L2 norm, beta and
// gate maps.  Prefill writes bf16 q, k, v and fp32 g, beta; the decode form is
// fused into the recurrent step.
struct PrologueArgs {
    const __nv_bfloat16* q_raw;
    const __nv_bfloat16* k_raw;
    const __nv_bfloat16* v_raw;
    const float* g_raw;
    const float* beta_raw;
    const float* conv_w;     // [H, 2 dk + dv, 4]
    float* ring;             // [B, H, 4, 2 dk + dv] or null
    const int* pos0;         // [B] or null (0)
    bool silu;
    __nv_bfloat16* q;
    __nv_bfloat16* k;
    __nv_bfloat16* v;
    float* g;
    float* beta;
    int B, T, H, dk, dv;
    bool per_channel;
};
cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream);

// The ring update of a prologue pass alone (slot (pos0 + t) mod 4 takes the
// raw input of token t for the last min(T, 4) tokens).
cudaError_t launch_prologue_ring(const PrologueArgs& a, cudaStream_t stream);

// The prefill with the prologue applied while loading the raw projections
// (pool form, dk = dv = 128, 2 * B * H <= #SMs), then the ring update.
// cudaErrorNotSupported when that form does not apply (nothing launched but,
// possibly, a memset of scratch); the caller then runs the two passes.
struct ProPrefill {
    PrologueArgs pro;          // raw inputs, taps, ring, pos0, activation (q..beta unused)
    const float* state_in;     // [B, H, dk, dv] or null
    float* state_out;          // [B, H, dk, dv] or null
    float* out;                // [B, T, H, dv] fp32
};
cudaError_t launch_chunk_pool_prologue(const ProPrefill& a, cudaStream_t stream);

struct StepPrologueArgs {
    const __nv_bfloat16* q_raw;
    const __nv_bfloat16* k_raw;
    const __nv_bfloat16* v_raw;
    const float* g_raw;
    const float* beta_raw;
    const float* conv_w;
    float* ring;
    const int* pos;          // [B] or null (0)
    bool silu;
    const float* state_in;
    float* state_out;
    float* out;              // [B, H, dv] fp32
    int B, H, dk, dv;
    bool per_channel;
};
cudaError_t launch_step_prologue(const StepPrologueArgs& a, cudaStream_t stream);

// Device status word written by kernels that abandon a bounded wait.
cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream);

}  // namespace gdn
