// KDA prefill on CUDA cores in fp32, token by token (every dtype, dk/dv in {64, 128}).
//
// This is the library's fp32 path (the bf16 tensor-core kernel cannot reach fp32
// accuracy) and the fallback kernel for head sizes the tensor-core kernel does not
// cover.  It runs the recurrence exactly as defined, one token at a time:
//   S <- Diag(exp g_t) S;  u = beta_t (v_t - S^T k_t);  S <- S + k_t u^T;  o_t = S^T q_t
// ("Day 21" course page, interview item D19 and quiz Q9), with fp32 arithmetic and the
// state held in registers for the whole sequence.
//
// The recurrence is separable over the dv columns of S (column c only ever mixes with
// v[c] and u[c]), so each CTA owns one (b, h) and a 32-column slice of the state: more
// CTAs for the same problem, and 16 state values per thread.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSlice = 32;                 // state columns per CTA
constexpr int kLpr = kSlice / 4;           // threads per row (float4 each) = 8
constexpr int kRpp = kSimtThreads / kLpr;  // rows per pass = 32

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads)
kda_prefill_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                        const Tin* __restrict__ g, const Tin* __restrict__ beta,
                        const float* S0, Tin* __restrict__ o, float* ST, int T_all, int H,
                        float* S_mid, int interval, int n_mid, const int* __restrict__ cu_seqlens, int* status,
                        int fused) {
    constexpr int RPT = DK / kRpp;  // rows per thread (4 or 2)
    constexpr int NW = kSimtThreads / 32;
    constexpr int NSLICE = DV / kSlice;

    __shared__ float qs[2][DK], ks[2][DK], es[2][DK], vs[2][kSlice], bs[2];
    __shared__ float4 red_a[NW][kLpr], red_b[NW][kLpr];
    __shared__ float4 us[kLpr];
    __shared__ float qss[2][DK / 32], kss[2][DK / 32];   // prologue: per-warp sums of q^2, k^2
    __shared__ float s_invk[2];                          // prologue: 1/|k| of the token

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c4 = tid % kLpr, rg = tid / kLpr;
    const int slice = blockIdx.x % NSLICE;
    const size_t bh = blockIdx.x / NSLICE;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int col0 = slice * kSlice;
    // tokens of this sequence: rows base .. base + T - 1 of the token axis
    size_t base = (size_t)b * T_all;
    int T = T_all;
    if (cu_seqlens) {
        // offsets that are not one valid layout (one overlapping or out-of-range sequence is
        // enough) leave every sequence empty and are reported
        const bool valid = packed_offsets_valid(cu_seqlens, (int)(gridDim.x / NSLICE / H), T_all);
        if (!valid && threadIdx.x == 0) report_status(status, KDA_ERR_INVALID_ARG);
        base = valid ? (size_t)cu_seqlens[b] : 0;
        T = valid ? cu_seqlens[b + 1] - cu_seqlens[b] : 0;
    }

    float4 s[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
        const int r = rg + j * kRpp;
        if (S0) s[j] = *reinterpret_cast<const float4*>(S0 + (bh * DK + r) * DV + col0 + 4 * c4);
        else s[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    auto stage = [&](int t, int buf) {
        const size_t row = (base + t) * H + h;
        if (tid < DK) {
            const float qv = load_elem(q, row * DK + tid), kv = load_elem(k, row * DK + tid);
            qs[buf][tid] = qv;
            ks[buf][tid] = kv;
            float gv = load_elem(g, row * DK + tid);
            if (fused) {
                // g = -5 sigmoid(z); the q and k norms as per-warp partial sums (full warps here)
                gv = -5.f / (1.f + expf(-gv));
                float sq = qv * qv, sk = kv * kv;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                if (lane == 0) { qss[buf][warp] = sq; kss[buf][warp] = sk; }
            }
            es[buf][tid] = expf(gv);
        } else if (tid < DK + kSlice) {
            vs[buf][tid - DK] = load_elem(v, row * DV + col0 + (tid - DK));
        } else if (tid == DK + kSlice) {
            const float bz = load_elem(beta, row);
            bs[buf] = fused ? 1.f / (1.f + expf(-bz)) : bz;
        }
    };

    if (T > 0) stage(0, 0);
    __syncthreads();
    for (int t = 0; t < T; ++t) {
        const int buf = t & 1;
        // decay, then the partial column sums S'^T k and S'^T q over this thread's rows
        float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int r = rg + j * kRpp;
            const float e = es[buf][r], kr = ks[buf][r], qr = qs[buf][r];
            s[j].x *= e; s[j].y *= e; s[j].z *= e; s[j].w *= e;
            pa.x += s[j].x * kr; pa.y += s[j].y * kr; pa.z += s[j].z * kr; pa.w += s[j].w * kr;
            pb.x += s[j].x * qr; pb.y += s[j].y * qr; pb.z += s[j].z * qr; pb.w += s[j].w * qr;
        }
#pragma unroll
        for (int off = kLpr; off < 32; off <<= 1) {
            pa.x += __shfl_xor_sync(0xffffffffu, pa.x, off); pa.y += __shfl_xor_sync(0xffffffffu, pa.y, off);
            pa.z += __shfl_xor_sync(0xffffffffu, pa.z, off); pa.w += __shfl_xor_sync(0xffffffffu, pa.w, off);
            pb.x += __shfl_xor_sync(0xffffffffu, pb.x, off); pb.y += __shfl_xor_sync(0xffffffffu, pb.y, off);
            pb.z += __shfl_xor_sync(0xffffffffu, pb.z, off); pb.w += __shfl_xor_sync(0xffffffffu, pb.w, off);
        }
        if (lane < kLpr) { red_a[warp][lane] = pa; red_b[warp][lane] = pb; }
        __syncthreads();
        // Every thread is past iteration t-1 here, so the other buffer is free: stage the
        // next token into it (read only after the second barrier below).
        if (t + 1 < T) stage(t + 1, buf ^ 1);
        if (warp == 0) {
            float kq = 0.f;
#pragma unroll
            for (int i = lane; i < DK; i += 32) kq += ks[buf][i] * qs[buf][i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
            // prologue: the sums above used the raw q and k; scale by 1/|q| and 1/|k|
            float inv_q = 1.f, inv_k = 1.f;
            if (fused) {
                float sq = 0.f, sk = 0.f;
#pragma unroll
                for (int w = 0; w < DK / 32; ++w) { sq += qss[buf][w]; sk += kss[buf][w]; }
                inv_q = sq > 0.f ? rsqrtf(sq) : 0.f;
                inv_k = sk > 0.f ? rsqrtf(sk) : 0.f;
                kq *= inv_q * inv_k;
                if (lane == 0) s_invk[buf] = inv_k;
            }
            if (lane < kLpr) {
                float4 a = red_a[0][lane], bb = red_b[0][lane];
#pragma unroll
                for (int w = 1; w < NW; ++w) {
                    const float4 ta = red_a[w][lane], tb = red_b[w][lane];
                    a.x += ta.x; a.y += ta.y; a.z += ta.z; a.w += ta.w;
                    bb.x += tb.x; bb.y += tb.y; bb.z += tb.z; bb.w += tb.w;
                }
                a.x *= inv_k; a.y *= inv_k; a.z *= inv_k; a.w *= inv_k;
                bb.x *= inv_q; bb.y *= inv_q; bb.z *= inv_q; bb.w *= inv_q;
                const float bt = bs[buf];
                float4 u;
                u.x = bt * (vs[buf][4 * lane + 0] - a.x);
                u.y = bt * (vs[buf][4 * lane + 1] - a.y);
                u.z = bt * (vs[buf][4 * lane + 2] - a.z);
                u.w = bt * (vs[buf][4 * lane + 3] - a.w);
                us[lane] = u;
                const size_t oo = ((base + t) * H + h) * DV + col0 + 4 * lane;
                store_elem(o, oo + 0, bb.x + kq * u.x);
                store_elem(o, oo + 1, bb.y + kq * u.y);
                store_elem(o, oo + 2, bb.z + kq * u.z);
                store_elem(o, oo + 3, bb.w + kq * u.w);
            }
        }
        __syncthreads();
        const float4 u = us[c4];
        const float kscale = fused ? s_invk[buf] : 1.f;
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const float kr = ks[buf][rg + j * kRpp] * kscale;
            s[j].x += kr * u.x; s[j].y += kr * u.y; s[j].z += kr * u.z; s[j].w += kr * u.w;
        }
        // the state after a multiple of the interval
        if (n_mid > 0 && (t + 1) % interval == 0) {
            const size_t base = bh * (size_t)n_mid + (size_t)((t + 1) / interval - 1);
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
                const int r = rg + j * kRpp;
                __stcs(reinterpret_cast<float4*>(S_mid + (base * DK + r) * DV + col0 + 4 * c4), s[j]);
            }
        }
    }
    if (ST) {
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int r = rg + j * kRpp;
            *reinterpret_cast<float4*>(ST + (bh * DK + r) * DV + col0 + 4 * c4) = s[j];
        }
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t s) {
    const unsigned grid = (unsigned)((size_t)a.B * a.H * (DV / kSlice));
    kda_prefill_simt_kernel<Tin, DK, DV><<<grid, kSimtThreads, 0, s>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
        static_cast<const Tin*>(a.g), static_cast<const Tin*>(a.beta), a.S0, static_cast<Tin*>(a.o),
        a.ST, a.T, a.H, a.S_mid, a.interval, a.n_mid, a.cu_seqlens, a.status, a.fused);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_dims(const PrefillArgs& a, cudaStream_t s) {
    if (a.dk == 128 && a.dv == 128) return launch_t<Tin, 128, 128>(a, s);
    if (a.dk == 128 && a.dv == 64) return launch_t<Tin, 128, 64>(a, s);
    if (a.dk == 64 && a.dv == 128) return launch_t<Tin, 64, 128>(a, s);
    return launch_t<Tin, 64, 64>(a, s);
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    if (a.dtype == KDA_DTYPE_BF16) return dispatch_dims<__nv_bfloat16>(a, s);
    return dispatch_dims<float>(a, s);
}

}  // namespace kda
