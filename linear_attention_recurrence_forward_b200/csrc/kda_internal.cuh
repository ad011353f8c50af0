// Internal declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Arguments of one prefill launch, already validated by the C ABI layer.
struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* g;
    const void* beta;
    const float* S0;  // may be null (zero state)
    void* o;
    float* ST;        // may be null
    int B, T, H, dk, dv;
    int dtype;        // kda_dtype
    int* status;      // device status word
    unsigned long long timeout_ns;  // limit of every device-side wait
    int skip_handoff;               // test hook: 1 = the prep group never signals its first hand-off
    float* S_mid;                   // states every `interval` tokens [B, H, n_mid, dk, dv], or null
    int interval;                   // multiple of 64 when S_mid is set
    int n_mid;                      // T / interval when S_mid is set, else 0
    // Packed variable-length sequences: when set, q, k, g, v, o are [T, H, d] with T the total
    // token count, B the number of sequences, and sequence b = tokens cu_seqlens[b] .. [b+1]-1
    // (device array of B + 1 ints, checked by the kernels).
    const int* cu_seqlens;
    // Gate and normalisation prologue: q and k are raw (each kernel L2-normalises them over the
    // head dimension), g holds the decay logit z (g = -5 sigmoid(z)) and beta the write logit
    // (beta = sigmoid)
    int fused;
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* g;
    const void* beta;
    float* S;
    void* o;
    int B, H, dk, dv;
    int dtype;
    int* status;
    // Paged states: when set, sequence b's state is S[slots[b]] of a pool of n_slots states per
    // head ([n_slots, H, dk, dv]); slots[b] < 0 skips the sequence.
    const int* slots;
    int n_slots;
};

// Launchers: return cudaSuccess or the launch error.  Defined in their kernel's .cu file.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
bool prefill_tc_supports(const PrefillArgs& a);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_state_compose(const float* M, const float* S, const float* N, float* out, int count, int dk,
                                 int dv, cudaStream_t s);
// o_out = o_in + per token S^T C (kda_output_correct; arguments validated by the caller)
cudaError_t launch_output_correct(const void* C, const float* S, const void* o_in, void* o_out, int B, int T, int H,
                                  int dk, int dv, int dtype, int* status, unsigned long long timeout_ns,
                                  cudaStream_t s);
// The driver's cuTensorMapEncodeTiled (looked up once), or null.
void* tensor_map_encoder();

// Element loads/stores for the two input dtypes.
__device__ __forceinline__ float load_elem(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Whether packed-sequence offsets form one valid layout, 0 <= cu[0] <= cu[1] <= ... <= cu[n] <= T
// (non-decreasing, so no two sequences share a token).  A block-wide vote: every thread of the
// block must call it, and all of them get the same answer.
__device__ __forceinline__ bool packed_offsets_valid(const int* cu, int n, int T) {
    bool ok = true;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int a = cu[i], b = cu[i + 1];
        ok = ok && a <= b && (i > 0 || a >= 0) && (i < n - 1 || b <= T);
    }
    return __syncthreads_and(ok) != 0;
}

// Set the device status word once (first error wins).
__device__ __forceinline__ void report_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace kda
