// C ABI of the KDA library: argument validation, kernel choice, the device status word.
//
// Everything here runs on the host before a launch; nothing is enqueued unless every
// check passes.  The kernels themselves live in kda_decode.cu, kda_prefill_simt.cu and
// kda_prefill_tc.cu.
#include <atomic>
#include <mutex>
#include <stdint.h>

#include "kda_internal.cuh"

// One status word per device (this module is loaded once per device context).  Kernels
// receive its device address as an argument and set it on a timed-out wait.
__device__ int g_kda_status_word = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per device-side wait
std::mutex g_mutex;
// Wait-timeout test hook (kda_debug_set_wait_fault); read at every tensor-core prefill launch.
std::atomic<int> g_skip_handoff{0};
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
int* g_status_addr[kMaxDevices] = {nullptr};

int* status_word_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_status_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_status_word) != cudaSuccess) return nullptr;
        g_status_addr[dev] = static_cast<int*>(p);
    }
    return g_status_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dim_ok(int d) { return d == 64 || d == 128; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void* p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

size_t elem_size(int dtype) { return dtype == KDA_DTYPE_BF16 ? 2 : 4; }

int validate_prefill(const void* q, const void* k, const void* v, const void* g, const void* beta,
                     const float* S0, const void* o, const float* ST, int B, int T, int H, int dk,
                     int dv, int dtype, int n_states = -1) {
    if (n_states < 0) n_states = B;   // states [n_states, H, dk, dv]
    if (B <= 0 || H <= 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    // 64-bit element counts must stay far from overflow
    const double elems = (double)B * (double)T * (double)H * (double)(dk > dv ? dk : dv);
    if (elems > 9.0e15) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, S0, o, ST};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if (T > 0) {
        const size_t es = elem_size(dtype);
        const size_t n_tok = (size_t)B * T * H;
        const Range ro = range_of(o, n_tok * dv * es);
        const Range ins[] = {range_of(q, n_tok * dk * es), range_of(k, n_tok * dk * es),
                             range_of(v, n_tok * dv * es), range_of(g, n_tok * dk * es),
                             range_of(beta, n_tok * es)};
        for (const Range& r : ins)
            if (overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
        const size_t sbytes = (size_t)n_states * H * dk * dv * sizeof(float);
        if (S0 && overlaps(ro, range_of(S0, sbytes))) return KDA_ERR_INVALID_ARG;
        if (ST) {
            const Range rs = range_of(ST, sbytes);
            if (overlaps(rs, ro)) return KDA_ERR_INVALID_ARG;
            for (const Range& r : ins)
                if (overlaps(rs, r)) return KDA_ERR_INVALID_ARG;
        }
    }
    if (S0 && ST && S0 != ST) {
        const size_t sbytes = (size_t)n_states * H * dk * dv * sizeof(float);
        if (overlaps(range_of(S0, sbytes), range_of(ST, sbytes))) return KDA_ERR_INVALID_ARG;
    }
    return KDA_OK;
}

// The intermediate-state output: interval, size, alignment, and no overlap with anything else.
int validate_states(const void* q, const void* k, const void* v, const void* g, const void* beta,
                    const float* S0, const void* o, const float* ST, const float* S_mid, int interval,
                    int B, int T, int H, int dk, int dv, int dtype, int* n_mid_out) {
    if (interval <= 0) return KDA_ERR_INVALID_ARG;
    if (interval % 64 != 0) return KDA_ERR_UNSUPPORTED;
    const int n_mid = T / interval;
    *n_mid_out = n_mid;
    if (n_mid == 0) return KDA_OK;
    if (!S_mid) return KDA_ERR_INVALID_ARG;
    if (!aligned16(S_mid)) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype);
    const size_t n_tok = (size_t)B * T * H;
    const size_t sbytes = (size_t)B * H * dk * dv * sizeof(float);
    const Range rm = range_of(S_mid, sbytes * (size_t)n_mid);
    const Range others[] = {range_of(q, n_tok * dk * es), range_of(k, n_tok * dk * es),
                            range_of(v, n_tok * dv * es), range_of(g, n_tok * dk * es),
                            range_of(beta, n_tok * es), range_of(o, n_tok * dv * es),
                            range_of(S0, S0 ? sbytes : 0), range_of(ST, ST ? sbytes : 0)};
    for (const Range& r : others)
        if (overlaps(rm, r)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

int forward_impl(const void* q, const void* k, const void* v, const void* g, const void* beta,
                 const float* S0, void* o, float* ST, int B, int T, int H, int dk, int dv, int dtype,
                 int impl, cudaStream_t stream, float* S_mid = nullptr, int interval = 0,
                 const int* cu_seqlens = nullptr, int fused = 0) {
    if (impl != KDA_IMPL_AUTO && impl != KDA_IMPL_TCGEN05 && impl != KDA_IMPL_SIMT)
        return KDA_ERR_INVALID_ARG;
    // packed sequences: the activations are one batch entry of T tokens, the states B entries
    int rc = cu_seqlens ? validate_prefill(q, k, v, g, beta, S0, o, ST, 1, T, H, dk, dv, dtype, B)
                        : validate_prefill(q, k, v, g, beta, S0, o, ST, B, T, H, dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (cu_seqlens) {
        if (!aligned16(cu_seqlens)) return KDA_ERR_MISALIGNED;
        const Range rc_ = range_of(cu_seqlens, (size_t)(B + 1) * sizeof(int));
        const size_t es = elem_size(dtype);
        if (T > 0 && overlaps(rc_, range_of(o, (size_t)T * H * dv * es))) return KDA_ERR_INVALID_ARG;
        if (ST && overlaps(rc_, range_of(ST, (size_t)B * H * dk * dv * sizeof(float)))) return KDA_ERR_INVALID_ARG;
    }
    int n_mid = 0;
    if (interval != 0 || S_mid) {
        rc = validate_states(q, k, v, g, beta, S0, o, ST, S_mid, interval, B, T, H, dk, dv, dtype, &n_mid);
        if (rc != KDA_OK) return rc;
    }
    kda::PrefillArgs a{q, k, v, g, beta, S0, o, ST, B, T, H, dk, dv, dtype, nullptr,
                       g_timeout_ns.load(), g_skip_handoff.load(), n_mid > 0 ? S_mid : nullptr,
                       interval, n_mid, cu_seqlens, fused};
    const bool tc_ok = kda::prefill_tc_supports(a);
    if (impl == KDA_IMPL_TCGEN05 && !tc_ok) return KDA_ERR_UNSUPPORTED;
    if (T == 0) {
        // No tokens: the final state is the initial state.
        if (!ST) return KDA_OK;
        const size_t sbytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = S0 ? (S0 == ST ? cudaSuccess
                                       : cudaMemcpyAsync(ST, S0, sbytes, cudaMemcpyDeviceToDevice, stream))
                           : cudaMemsetAsync(ST, 0, sbytes, stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    a.status = status_word_for_current_device();
    if (!a.status) return KDA_ERR_CUDA;
    cudaError_t e;
    if (impl == KDA_IMPL_SIMT || (impl == KDA_IMPL_AUTO && !tc_ok)) e = kda::launch_prefill_simt(a, stream);
    else e = kda::launch_prefill_tc(a, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int decode_impl(const void* q, const void* k, const void* v, const void* g, const void* beta, float* S,
                int n_slots, const int* slots, void* o, int B, int H, int dk, int dv, int dtype,
                cudaStream_t stream) {
    if (B <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    if ((double)B * (double)H > 2.0e9) return KDA_ERR_INVALID_ARG;
    if (slots && (n_slots <= 0 || (double)n_slots * (double)H > 2.0e9)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, S, o, slots ? (const void*)slots : (const void*)q};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype);
    const size_t n = (size_t)B * H;
    const size_t n_state = slots ? (size_t)n_slots * H : n;
    const Range rs = range_of(S, n_state * dk * dv * sizeof(float));
    const Range ro = range_of(o, n * dv * es);
    const Range ins[] = {range_of(q, n * dk * es), range_of(k, n * dk * es), range_of(v, n * dv * es),
                         range_of(g, n * dk * es), range_of(beta, n * es)};
    if (overlaps(rs, ro)) return KDA_ERR_INVALID_ARG;
    for (const Range& r : ins)
        if (overlaps(rs, r) || overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
    if (slots) {
        const Range rt = range_of(slots, (size_t)B * sizeof(int));
        if (overlaps(rt, rs) || overlaps(rt, ro)) return KDA_ERR_INVALID_ARG;
    }
    kda::DecodeArgs a{q, k, v, g, beta, S, o, B, H, dk, dv, dtype, status_word_for_current_device(), slots,
                      n_slots};
    if (!a.status) return KDA_ERR_CUDA;
    return kda::launch_decode(a, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

int kda_forward_chunked(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv,
                        int dtype, struct CUstream_st* stream) {
    return forward_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, dtype, KDA_IMPL_AUTO, stream);
}

int kda_forward_chunked_impl(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* S0, void* o, float* S_T, int B, int T,
                             int H, int dk, int dv, int dtype, int impl, struct CUstream_st* stream) {
    return forward_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, dtype, impl, stream);
}

int kda_forward_chunked_states(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* S0, void* o, float* S_T,
                               float* S_mid, int interval, int B, int T, int H, int dk, int dv,
                               int dtype, int impl, struct CUstream_st* stream) {
    if (interval <= 0) return KDA_ERR_INVALID_ARG;
    return forward_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, dtype, impl, stream, S_mid,
                        interval);
}

int kda_forward_chunked_fused(const void* q_raw, const void* k_raw, const void* v, const void* z_g,
                              const void* z_beta, const float* S0, void* o, float* S_T, int B, int T, int H,
                              int dk, int dv, int dtype, int impl, struct CUstream_st* stream) {
    return forward_impl(q_raw, k_raw, v, z_g, z_beta, S0, o, S_T, B, T, H, dk, dv, dtype, impl, stream, nullptr,
                        0, nullptr, 1);
}

int kda_forward_varlen(const void* q, const void* k, const void* v, const void* g, const void* beta,
                       const int* cu_seqlens, const float* S0, void* o, float* S_T, int N, int T_total,
                       int H, int dk, int dv, int dtype, int impl, struct CUstream_st* stream) {
    if (N <= 0 || !cu_seqlens) return KDA_ERR_INVALID_ARG;
    return forward_impl(q, k, v, g, beta, S0, o, S_T, N, T_total, H, dk, dv, dtype, impl, stream, nullptr, 0,
                        cu_seqlens);
}

int kda_decode_step(const void* q, const void* k, const void* v, const void* g, const void* beta,
                    float* S, void* o, int B, int H, int dk, int dv, int dtype,
                    struct CUstream_st* stream) {
    return decode_impl(q, k, v, g, beta, S, 0, nullptr, o, B, H, dk, dv, dtype, stream);
}

int kda_decode_step_paged(const void* q, const void* k, const void* v, const void* g, const void* beta,
                          float* S_pool, int n_slots, const int* slots, void* o, int B, int H, int dk,
                          int dv, int dtype, struct CUstream_st* stream) {
    if (!slots) return KDA_ERR_INVALID_ARG;
    return decode_impl(q, k, v, g, beta, S_pool, n_slots, slots, o, B, H, dk, dv, dtype, stream);
}

int kda_state_compose(const float* M, const float* S_in, const float* N, float* S_out, int count, int dk,
                      int dv, struct CUstream_st* stream) {
    if (count <= 0) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (!M || !S_in || !S_out) return KDA_ERR_INVALID_ARG;
    if ((double)count * dk * (dk > dv ? dk : dv) > 9.0e15) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {M, S_in, N, S_out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t sbytes = (size_t)count * dk * dv * sizeof(float);
    const Range rm = range_of(M, (size_t)count * dk * dk * sizeof(float));
    const Range ro = range_of(S_out, sbytes);
    if (overlaps(rm, ro)) return KDA_ERR_INVALID_ARG;
    // S_out may be S_in or N exactly; any other overlap is not allowed
    if (S_out != S_in && overlaps(ro, range_of(S_in, sbytes))) return KDA_ERR_INVALID_ARG;
    if (N && S_out != N && overlaps(ro, range_of(N, sbytes))) return KDA_ERR_INVALID_ARG;
    return kda::launch_state_compose(M, S_in, N, S_out, count, dk, dv, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_get_device_status(struct CUstream_st* stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    int* addr = status_word_for_current_device();
    if (!addr) return KDA_ERR_CUDA;
    int value = 0;
    if (cudaMemcpy(&value, addr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(addr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
    return value;
}

const char* kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        default: return "KDA_ERR_UNKNOWN";
    }
}

int kda_version(void) { return 100; }

int kda_debug_set_wait_fault(int mode, unsigned long long timeout_ns) {
    if (mode != 0 && mode != 1) return KDA_ERR_INVALID_ARG;
    if (mode == 1 && (timeout_ns < 1000000ull || timeout_ns > 10000000000ull)) return KDA_ERR_INVALID_ARG;
    g_skip_handoff.store(mode);
    g_timeout_ns.store(mode ? timeout_ns : kDefaultTimeoutNs);
    return KDA_OK;
}

}  // extern "C"
