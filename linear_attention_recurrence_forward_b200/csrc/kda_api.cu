// C ABI of the KDA library: argument validation, kernel choice, the device status word, and
// the host-buffer prefill (copy-in, kernels and copy-out pipelined over segments).
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
    // AUTO: the chunkwise tensor-core kernel for bf16 (every supported head size), the fp32 kernel
    // for fp32 inputs; a bf16 shape the tensor-core kernel did not cover would be refused rather than
    // sent to the token-serial kernel behind the caller's back (KDA_IMPL_SIMT runs it when asked for)
    if (impl == KDA_IMPL_AUTO && dtype == KDA_DTYPE_BF16 && !tc_ok) return KDA_ERR_UNSUPPORTED;
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
    if (impl == KDA_IMPL_SIMT || (impl == KDA_IMPL_AUTO && dtype == KDA_DTYPE_FP32)) e = kda::launch_prefill_simt(a, stream);
    else e = kda::launch_prefill_tc(a, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ------------------------------------------------------------------ host-buffer prefill
//
// The work is cut into segments of one batch entry and at most kHostSegTokens tokens (a
// multiple of the 64-token chunk, so the chunking is that of the whole sequence).  Segment i
// uses activation slot i % 2 of the workspace and batch entry b the state slot b % 2, which
// carries the fp32 state from one segment of b to the next (the kernel updates it in place).
// Three streams overlap the copy-in of segment i+1 and the copy-out of segment i-1 with the
// kernel of segment i: inputs go in on one internal stream, the kernels run on the caller's
// stream, outputs come out on a second internal stream, ordered by events.
constexpr int kHostSegTokens = 2048;

size_t round_up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct HostPlan {
    int L;                                  // tokens per segment (the last one of a sequence may be shorter)
    size_t q, v, beta;                      // bytes of a slot's q (= k = g), v (= o) and beta buffers
    size_t slot, state, total;
};

HostPlan host_plan(int T, int H, int dk, int dv, int dtype) {
    HostPlan p{};
    const size_t es = elem_size(dtype);
    p.L = T < kHostSegTokens ? T : kHostSegTokens;
    const size_t n = (size_t)p.L * H;
    p.q = round_up256(n * dk * es);
    p.v = round_up256(n * dv * es);
    p.beta = round_up256(n * es);
    p.slot = 3 * p.q + 2 * p.v + p.beta;
    p.state = round_up256((size_t)H * dk * dv * sizeof(float));
    p.total = 2 * p.slot + 2 * p.state;
    return p;
}

int validate_host(const void* q, const void* k, const void* v, const void* g, const void* beta,
                  const float* S0, const void* o, const float* ST, int B, int T, int H, int dk, int dv,
                  int dtype, const void* ws, size_t ws_bytes, int impl) {
    if (impl != KDA_IMPL_AUTO && impl != KDA_IMPL_TCGEN05 && impl != KDA_IMPL_SIMT) return KDA_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    const double elems = (double)B * (double)T * (double)H * (double)(dk > dv ? dk : dv);
    if (elems > 9.0e15) return KDA_ERR_INVALID_ARG;
    if (!ws) return KDA_ERR_INVALID_ARG;
    if (!aligned16(ws)) return KDA_ERR_MISALIGNED;
    if (ws_bytes < host_plan(T, H, dk, dv, dtype).total) return KDA_ERR_INVALID_ARG;
    // the host buffers: outputs overlap no input (S_T may be S0 itself)
    const size_t es = elem_size(dtype);
    const size_t n_tok = (size_t)B * T * H;
    const size_t sbytes = (size_t)B * H * dk * dv * sizeof(float);
    const Range ins[] = {range_of(q, T ? n_tok * dk * es : 0), range_of(k, T ? n_tok * dk * es : 0),
                         range_of(v, T ? n_tok * dv * es : 0), range_of(g, T ? n_tok * dk * es : 0),
                         range_of(beta, T ? n_tok * es : 0)};
    const Range ro = range_of(o, T ? n_tok * dv * es : 0);
    for (const Range& r : ins)
        if (overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
    if (S0 && overlaps(ro, range_of(S0, sbytes))) return KDA_ERR_INVALID_ARG;
    if (ST) {
        const Range rs = range_of(ST, sbytes);
        if (overlaps(rs, ro)) return KDA_ERR_INVALID_ARG;
        for (const Range& r : ins)
            if (overlaps(rs, r)) return KDA_ERR_INVALID_ARG;
        if (S0 && S0 != ST && overlaps(rs, range_of(S0, sbytes))) return KDA_ERR_INVALID_ARG;
    }
    return KDA_OK;
}

int forward_host_impl(const void* q, const void* k, const void* v, const void* g, const void* beta,
                      const float* S0, void* o, float* ST, int B, int T, int H, int dk, int dv, int dtype,
                      void* ws, size_t ws_bytes, int impl, cudaStream_t stream) {
    int rc = validate_host(q, k, v, g, beta, S0, o, ST, B, T, H, dk, dv, dtype, ws, ws_bytes, impl);
    if (rc != KDA_OK) return rc;
    const HostPlan P = host_plan(T, H, dk, dv, dtype);
    const size_t es = elem_size(dtype);
    const size_t sbytes = (size_t)H * dk * dv * sizeof(float);
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* state[2] = {reinterpret_cast<float*>(base + 2 * P.slot),
                       reinterpret_cast<float*>(base + 2 * P.slot + P.state)};
    if (T == 0) {
        // no tokens: S_T = S0 (or zeros), through a state slot, in order on the caller's stream
        if (!ST) return KDA_OK;
        for (int b = 0; b < B; ++b) {
            cudaError_t e = S0 ? cudaMemcpyAsync(state[0], S0 + (size_t)b * H * dk * dv, sbytes,
                                                 cudaMemcpyHostToDevice, stream)
                               : cudaMemsetAsync(state[0], 0, sbytes, stream);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(ST + (size_t)b * H * dk * dv, state[0], sbytes, cudaMemcpyDeviceToHost, stream);
            if (e != cudaSuccess) return KDA_ERR_CUDA;
        }
        return KDA_OK;
    }
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[8] = {};   // start, in[2], done[2], out[2], end
    bool ok = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; i < 8 && ok; ++i) ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
    cudaEvent_t ev_start = ev[0], ev_end = ev[7];
    cudaEvent_t ev_in[2] = {ev[1], ev[2]}, ev_done[2] = {ev[3], ev[4]}, ev_out[2] = {ev[5], ev[6]};
    // everything this call enqueues follows the work already on the caller's stream
    if (ok) ok = cudaEventRecord(ev_start, stream) == cudaSuccess &&
                 cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess;
    auto h2d = [&](void* dst, const void* src, size_t n) {
        if (ok) ok = cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s_in) == cudaSuccess;
    };
    auto d2h = [&](void* dst, const void* src, size_t n) {
        if (ok) ok = cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
    };
    bool out_pending[2] = {false, false};
    int seg = 0;
    for (int b = 0; b < B && ok && rc == KDA_OK; ++b) {
        float* Sb = state[b & 1];
        for (int t0 = 0; t0 < T && ok && rc == KDA_OK; t0 += P.L, ++seg) {
            const int L = T - t0 < P.L ? T - t0 : P.L;
            const int s = seg & 1;
            uint8_t* sl = base + (size_t)s * P.slot;
            uint8_t *dq = sl, *dk_ = sl + P.q, *dg = sl + 2 * P.q, *dv_ = sl + 3 * P.q;
            uint8_t *dbeta = dv_ + P.v, *do_ = dbeta + P.beta;
            const size_t th = ((size_t)b * T + t0) * H;   // first token-head of the segment
            const size_t n = (size_t)L * H;
            // copy-in: the slot (and the state slot of batch entry b - 2) is free once the segment
            // two back has been copied out
            if (out_pending[s] && ok) ok = cudaStreamWaitEvent(s_in, ev_out[s], 0) == cudaSuccess;
            h2d(dq, static_cast<const uint8_t*>(q) + th * dk * es, n * dk * es);
            h2d(dk_, static_cast<const uint8_t*>(k) + th * dk * es, n * dk * es);
            h2d(dg, static_cast<const uint8_t*>(g) + th * dk * es, n * dk * es);
            h2d(dv_, static_cast<const uint8_t*>(v) + th * dv * es, n * dv * es);
            h2d(dbeta, static_cast<const uint8_t*>(beta) + th * es, n * es);
            if (t0 == 0 && S0) h2d(Sb, S0 + (size_t)b * H * dk * dv, sbytes);
            if (ok) ok = cudaEventRecord(ev_in[s], s_in) == cudaSuccess &&
                         cudaStreamWaitEvent(stream, ev_in[s], 0) == cudaSuccess;
            if (!ok) break;
            // the prefill of the segment, from the carried state (or S0 / zeros at the start)
            const float* s_from = (t0 == 0 && !S0) ? nullptr : Sb;
            rc = forward_impl(dq, dk_, dv_, dg, dbeta, s_from, do_, Sb, 1, L, H, dk, dv, dtype, impl, stream);
            if (rc != KDA_OK) break;
            ok = cudaEventRecord(ev_done[s], stream) == cudaSuccess &&
                 cudaStreamWaitEvent(s_out, ev_done[s], 0) == cudaSuccess;
            // copy-out of o, and of the final state after the last segment of b
            d2h(static_cast<uint8_t*>(o) + th * dv * es, do_, n * dv * es);
            if (ST && t0 + L == T) d2h(ST + (size_t)b * H * dk * dv, Sb, sbytes);
            if (ok) ok = cudaEventRecord(ev_out[s], s_out) == cudaSuccess;
            out_pending[s] = true;
        }
    }
    // the caller's stream continues only after every copy-out (also after a failure part-way)
    if (ev_end && s_out && cudaEventRecord(ev_end, s_out) == cudaSuccess)
        (void)cudaStreamWaitEvent(stream, ev_end, 0);
    for (cudaEvent_t e : ev)
        if (e) cudaEventDestroy(e);   // released once complete
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    if (rc != KDA_OK) return rc;
    return ok ? KDA_OK : KDA_ERR_CUDA;
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

size_t kda_forward_chunked_host_workspace(int T, int H, int dk, int dv, int dtype) {
    if (T < 0 || H <= 0 || !head_dim_ok(dk) || !head_dim_ok(dv) ||
        (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32))
        return 0;
    return host_plan(T, H, dk, dv, dtype).total;
}

int kda_forward_chunked_host(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv,
                             int dtype, void* workspace, size_t workspace_bytes, int impl, cudaStream_t stream) {
    return forward_host_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, dtype, workspace, workspace_bytes,
                             impl, stream);
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

int kda_output_correct(const void* C, const float* S_in, const void* o_in, void* o_out, int B, int T, int H, int dk,
                       int dv, int dtype, struct CUstream_st* stream) {
    if (B <= 0 || H <= 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((double)B * (double)T * (double)H * (double)(dk > dv ? dk : dv) > 9.0e15) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    if (!C || !S_in || !o_in || !o_out) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {C, S_in, o_in, o_out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype);
    const size_t n_tok = (size_t)B * T * H;
    const Range ro = range_of(o_out, n_tok * dv * es);
    const Range rc = range_of(C, n_tok * dk * es);
    const Range rs = range_of(S_in, (size_t)B * H * dk * dv * sizeof(float));
    // o_out may be o_in itself (in place); no other overlap
    if (overlaps(ro, rc) || overlaps(ro, rs)) return KDA_ERR_INVALID_ARG;
    if (o_out != o_in && overlaps(ro, range_of(o_in, n_tok * dv * es))) return KDA_ERR_INVALID_ARG;
    int* status = status_word_for_current_device();
    if (!status) return KDA_ERR_CUDA;
    return kda::launch_output_correct(C, S_in, o_in, o_out, B, T, H, dk, dv, dtype, status, g_timeout_ns.load(),
                                      stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
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
