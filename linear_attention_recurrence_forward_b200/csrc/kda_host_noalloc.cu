// Host-buffer prefill that allocates nothing: kda_forward_chunked_host_noalloc.
//
// kda_forward_chunked_host needs a device workspace from its caller.  Some callers have no way to
// provide one: a host application that hands the library plain host arrays through a C foreign-
// function interface and holds no CUDA allocator of its own, or an engine whose device memory is
// entirely owned by a pool that forbids allocations outside it (cudaMalloc there would also
// synchronise the device in the middle of latency-critical work).  This entry point stages the
// work through one fixed scratch array that the library itself reserves in device memory when it
// is loaded, so the caller passes only host buffers and a stream, and no call allocates.
//
// Everything runs in order on the caller's stream: copy one segment's inputs in, run the prefill
// on it, copy its outputs out, next segment.  The segment length is the largest multiple of the
// 64-token chunk whose inputs, outputs and one carried state fit the scratch, so the chunking and
// the state carried between segments (fp32, in device memory) are those of a single prefill over
// the whole sequence.
#include <mutex>
#include <stdint.h>

#include "kda_internal.cuh"

// The fixed scratch: one segment's q, k, g, v, beta and o plus one fp32 state slot [H, dk, dv].
// Every device that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
unsigned char* g_scratch_addr[kMaxDevices] = {nullptr};

size_t round_up256(size_t x) { return (x + 255) & ~(size_t)255; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }
size_t elem_size(int dtype) { return dtype == KDA_DTYPE_BF16 ? 2 : 4; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void* p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

// Layout of the scratch for one call: the state slot first, then a segment of L tokens.
struct Plan {
    int L;                    // tokens per segment (0: the problem does not fit)
    size_t state, q, v, beta; // bytes of the state slot and of one segment's q (= k = g), v (= o), beta
};

Plan make_plan(int T, int H, int dk, int dv, int dtype) {
    Plan p{};
    const size_t es = elem_size(dtype);
    p.state = round_up256((size_t)H * dk * dv * sizeof(float));
    auto bytes = [&](size_t L) {
        const size_t n = L * (size_t)H;
        return p.state + 3 * round_up256(n * dk * es) + 2 * round_up256(n * dv * es) + round_up256(n * es);
    };
    const size_t cap = KDA_NOALLOC_SCRATCH_BYTES;
    size_t L = 0;
    if (T > 0 && T <= 64) {
        L = bytes((size_t)T) <= cap ? (size_t)T : 0;
    } else if (T > 64) {
        // the largest multiple of 64 that fits (and is not longer than needed)
        const size_t per_tok = (size_t)H * (3 * dk * es + 2 * dv * es + es);
        L = cap > p.state ? ((cap - p.state) / per_tok) & ~(size_t)63 : 0;
        if (L > (size_t)((T + 63) & ~63)) L = (size_t)((T + 63) & ~63);
        while (L >= 64 && bytes(L) > cap) L -= 64;   // the 256-byte rounding of the six buffers
    }
    p.L = (int)L;
    const size_t n = L * (size_t)H;
    p.q = round_up256(n * dk * es);
    p.v = round_up256(n * dv * es);
    p.beta = round_up256(n * es);
    return p;
}

// The scratch's device address on the current device (host code must not use the symbol itself:
// in host code it names a host-side stand-in).  Looked up once per device.
unsigned char* scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = static_cast<unsigned char*>(p);
    }
    return g_scratch_addr[dev];
}

int validate(const void* q, const void* k, const void* v, const void* g, const void* beta, const float* S0,
             const void* o, const float* ST, int B, int T, int H, int dk, int dv, int dtype, int impl) {
    if (impl != KDA_IMPL_AUTO && impl != KDA_IMPL_TCGEN05 && impl != KDA_IMPL_SIMT) return KDA_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16 && dtype != KDA_DTYPE_FP32) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    // the kernel choice of kda_forward_chunked_impl, checked here so that a refusal comes before
    // any copy is enqueued
    const bool tc_shape = dtype == KDA_DTYPE_BF16;   // head sizes 64 and 128 both (checked above)
    if (impl == KDA_IMPL_TCGEN05 && !tc_shape) return KDA_ERR_UNSUPPORTED;
    if (impl == KDA_IMPL_AUTO && dtype == KDA_DTYPE_BF16 && !tc_shape) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    if ((double)B * (double)T * (double)H * (double)(dk > dv ? dk : dv) > 9.0e15) return KDA_ERR_INVALID_ARG;
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

}  // namespace

extern "C" int kda_forward_chunked_host_noalloc(const void* q, const void* k, const void* v, const void* g,
                                                const void* beta, const float* S0, void* o, float* S_T, int B,
                                                int T, int H, int dk, int dv, int dtype, int impl,
                                                struct CUstream_st* stream) {
    int rc = validate(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, dtype, impl);
    if (rc != KDA_OK) return rc;
    const Plan P = make_plan(T, H, dk, dv, dtype);
    if (T > 0 && P.L == 0) return KDA_ERR_UNSUPPORTED;   // not even one chunk fits the fixed scratch
    if (P.state > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;
    unsigned char* base = scratch_for_current_device();
    if (!base) return KDA_ERR_CUDA;
    cudaStream_t s = stream;
    const size_t es = elem_size(dtype);
    const size_t sbytes = (size_t)H * dk * dv * sizeof(float);
    float* state = reinterpret_cast<float*>(base);
    unsigned char* dq = base + P.state;
    unsigned char *dk_ = dq + P.q, *dg = dk_ + P.q, *dv_ = dg + P.q, *dbeta = dv_ + P.v, *do_ = dbeta + P.beta;
    for (int b = 0; b < B; ++b) {
        const float* s0b = S0 ? S0 + (size_t)b * H * dk * dv : nullptr;
        float* stb = S_T ? S_T + (size_t)b * H * dk * dv : nullptr;
        if (T == 0) {
            // no tokens: S_T = S0 (or zeros), through the state slot
            if (!stb) continue;
            cudaError_t e = s0b ? cudaMemcpyAsync(state, s0b, sbytes, cudaMemcpyHostToDevice, s)
                                : cudaMemsetAsync(state, 0, sbytes, s);
            if (e == cudaSuccess) e = cudaMemcpyAsync(stb, state, sbytes, cudaMemcpyDeviceToHost, s);
            if (e != cudaSuccess) return KDA_ERR_CUDA;
            continue;
        }
        for (int t0 = 0; t0 < T; t0 += P.L) {
            const int L = T - t0 < P.L ? T - t0 : P.L;
            const size_t th = ((size_t)b * T + t0) * H;   // first token-head of the segment
            const size_t n = (size_t)L * H;
            cudaError_t e = cudaSuccess;
            auto h2d = [&](void* dst, const void* src, size_t bytes) {
                if (e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s);
            };
            h2d(dq, static_cast<const unsigned char*>(q) + th * dk * es, n * dk * es);
            h2d(dk_, static_cast<const unsigned char*>(k) + th * dk * es, n * dk * es);
            h2d(dg, static_cast<const unsigned char*>(g) + th * dk * es, n * dk * es);
            h2d(dv_, static_cast<const unsigned char*>(v) + th * dv * es, n * dv * es);
            h2d(dbeta, static_cast<const unsigned char*>(beta) + th * es, n * es);
            if (t0 == 0 && s0b) h2d(state, s0b, sbytes);
            if (e != cudaSuccess) return KDA_ERR_CUDA;
            // the first segment starts from S0 (or zeros: the kernels take a null S0 as zeros, so
            // nothing left in the scratch by an earlier call is read); later ones from the carried state
            const float* from = (t0 == 0 && !s0b) ? nullptr : state;
            rc = kda_forward_chunked_impl(dq, dk_, dv_, dg, dbeta, from, do_, state, 1, L, H, dk, dv, dtype, impl,
                                          stream);
            if (rc != KDA_OK) return rc;
            e = cudaMemcpyAsync(static_cast<unsigned char*>(o) + th * dv * es, do_, n * dv * es,
                                cudaMemcpyDeviceToHost, s);
            if (e == cudaSuccess && stb && t0 + L == T) e = cudaMemcpyAsync(stb, state, sbytes, cudaMemcpyDeviceToHost, s);
            if (e != cudaSuccess) return KDA_ERR_CUDA;
        }
    }
    return KDA_OK;
}
