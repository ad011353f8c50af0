// KDA single-token decode: the memory-bound fp32 state read-modify-write.
//
// Per (b, h), with S in R^{dk x dv} (fp32, row-major, updated in place):
//   S' = Diag(exp g) S;   a = S'^T k;   b = S'^T q;   u = beta (v - a);
//   o  = b + (k . q) u    (= S_new^T q, since S_new = S' + k u^T);   S_new = S' + k u^T.
// This is the recurrence of the "Day 21" course page (interview item D19, quiz Q9) for one
// token; the same page (item D17, quiz Q5) is why it is memory-bound: every state
// element is read and written once for ~7 flops.
//
// Design: the update is independent per value column (u_j and o_j need column j of the state and
// the scalar k . q only), so a state is split over CTAs by columns: one CTA of 256 threads per
// (state, 64-column slice), with no exchange between the slices.  That keeps 32 state values per
// thread, so several CTAs share an SM and one CTA's reductions overlap the others' loads and
// stores.  Lanes run along the columns with 16-byte vectors, so each warp instruction reads or
// writes whole contiguous row segments (coalesced); the state stays in registers between the
// read and the write (one pass, no re-read).  Column sums over dk use warp shuffles and one
// shared-memory step across warps.  Loads/stores use the evict-first streaming hints: a state
// is touched exactly once per step.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecodeThreads = 256;

constexpr int kSliceCols = 64;   // state columns per CTA

// DV: the state's columns (row stride); DVC: the columns of one CTA's slice
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads)
kda_decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                  const Tin* __restrict__ g, const Tin* __restrict__ beta, float* __restrict__ S,
                  Tin* __restrict__ o, int H, const int* __restrict__ slots, int n_slots, int* status) {
    constexpr int DVC = DV < kSliceCols ? DV : kSliceCols;
    constexpr int NSL = DV / DVC;                  // slices per state
    constexpr int LPR = DVC / 4;                   // threads per state row segment (float4 each)
    constexpr int RPP = kDecodeThreads / LPR;      // rows covered per pass
    constexpr int RPT = DK / RPP;                  // rows per thread
    constexpr int WPR = 32 / LPR;                  // rows per warp instruction (1 or 2)
    constexpr int NW = kDecodeThreads / 32;
    static_assert(RPT * RPP == DK && RPT >= 1, "bad decode tiling");

    __shared__ float qs[DK], ks[DK], es[DK];
    __shared__ float4 red_a[NW][LPR], red_b[NW][LPR];
    __shared__ float4 us[LPR];

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int c4 = tid % LPR, rg = tid / LPR;
    const size_t bh = blockIdx.x / NSL;
    const int col0 = (int)(blockIdx.x % NSL) * DVC;   // first column of this CTA's slice
    size_t sidx = bh;   // state of this (b, h): S[b, h], or S[slots[b], h] of a pool
    if (slots) {
        const int sl = slots[bh / H];
        if (sl < 0) return;                        // inactive sequence: nothing is read or written
        if (sl >= n_slots) {
            if (tid == 0) report_status(status, KDA_ERR_INVALID_ARG);
            return;
        }
        sidx = (size_t)sl * H + bh % H;
    }
    float4* Sv = reinterpret_cast<float4*>(S + sidx * DK * DV + col0);
    constexpr int RS = DV / 4;                     // float4s per full state row

    // Issue the state loads first: 16 B per thread per row, all independent.
    float4 s[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) s[j] = __ldcs(Sv + (size_t)(rg + j * RPP) * RS + c4);

    if (tid < DK) {
        qs[tid] = load_elem(q, bh * DK + tid);
        ks[tid] = load_elem(k, bh * DK + tid);
        es[tid] = expf(load_elem(g, bh * DK + tid));
    }
    __syncthreads();

    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
        const int r = rg + j * RPP;
        const float e = es[r], kr = ks[r], qr = qs[r];
        s[j].x *= e; s[j].y *= e; s[j].z *= e; s[j].w *= e;
        pa.x += s[j].x * kr; pa.y += s[j].y * kr; pa.z += s[j].z * kr; pa.w += s[j].w * kr;
        pb.x += s[j].x * qr; pb.y += s[j].y * qr; pb.z += s[j].z * qr; pb.w += s[j].w * qr;
    }
    // Combine the row groups that share a warp (lanes c4 and c4 + LPR when LPR == 16).
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        pa.x += __shfl_xor_sync(0xffffffffu, pa.x, off); pa.y += __shfl_xor_sync(0xffffffffu, pa.y, off);
        pa.z += __shfl_xor_sync(0xffffffffu, pa.z, off); pa.w += __shfl_xor_sync(0xffffffffu, pa.w, off);
        pb.x += __shfl_xor_sync(0xffffffffu, pb.x, off); pb.y += __shfl_xor_sync(0xffffffffu, pb.y, off);
        pb.z += __shfl_xor_sync(0xffffffffu, pb.z, off); pb.w += __shfl_xor_sync(0xffffffffu, pb.w, off);
    }
    (void)WPR;
    if (lane < LPR) { red_a[warp][lane] = pa; red_b[warp][lane] = pb; }
    __syncthreads();

    if (warp == 0) {
        // k . q over dk with a warp-shuffle reduction.
        float kq = 0.f;
#pragma unroll
        for (int i = lane; i < DK; i += 32) kq += ks[i] * qs[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane < LPR) {
            float4 a = red_a[0][lane], b = red_b[0][lane];
#pragma unroll
            for (int w = 1; w < NW; ++w) {
                const float4 ta = red_a[w][lane], tb = red_b[w][lane];
                a.x += ta.x; a.y += ta.y; a.z += ta.z; a.w += ta.w;
                b.x += tb.x; b.y += tb.y; b.z += tb.z; b.w += tb.w;
            }
            const float bt = load_elem(beta, bh);
            const size_t vo = bh * DV + col0 + 4 * lane;
            float4 u;
            u.x = bt * (load_elem(v, vo + 0) - a.x);
            u.y = bt * (load_elem(v, vo + 1) - a.y);
            u.z = bt * (load_elem(v, vo + 2) - a.z);
            u.w = bt * (load_elem(v, vo + 3) - a.w);
            us[lane] = u;
            store_elem(o, vo + 0, b.x + kq * u.x);
            store_elem(o, vo + 1, b.y + kq * u.y);
            store_elem(o, vo + 2, b.z + kq * u.z);
            store_elem(o, vo + 3, b.w + kq * u.w);
        }
    }
    __syncthreads();

    const float4 u = us[c4];
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
        const float kr = ks[rg + j * RPP];
        s[j].x += kr * u.x; s[j].y += kr * u.y; s[j].z += kr * u.z; s[j].w += kr * u.w;
        __stcs(Sv + (size_t)(rg + j * RPP) * RS + c4, s[j]);
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
    constexpr int nsl = DV < kSliceCols ? 1 : DV / kSliceCols;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * nsl);
    kda_decode_kernel<Tin, DK, DV><<<grid, kDecodeThreads, 0, s>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
        static_cast<const Tin*>(a.g), static_cast<const Tin*>(a.beta), a.S, static_cast<Tin*>(a.o), a.H, a.slots,
        a.n_slots, a.status);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_dims(const DecodeArgs& a, cudaStream_t s) {
    if (a.dk == 128 && a.dv == 128) return launch_decode_t<Tin, 128, 128>(a, s);
    if (a.dk == 128 && a.dv == 64) return launch_decode_t<Tin, 128, 64>(a, s);
    if (a.dk == 64 && a.dv == 128) return launch_decode_t<Tin, 64, 128>(a, s);
    return launch_decode_t<Tin, 64, 64>(a, s);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    if (a.dtype == KDA_DTYPE_BF16) return dispatch_dims<__nv_bfloat16>(a, s);
    return dispatch_dims<float>(a, s);
}

}  // namespace kda
