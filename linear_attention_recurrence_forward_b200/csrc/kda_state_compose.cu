// Composition of state maps for a sequence split over ranks: S_out = M S_in + N per head.
//
// Across a segment of tokens the recurrence is affine in its initial state,
// S_end = M S_start + N, with M = prod_t (I - beta_t k_t k_t^T) Diag(exp g_t) (dk x dk) and
// N the segment's final state from a zero start.  Only this fixed-size pair has to cross a
// sequence split, which is what KDA context parallelism exchanges (channel post on the K3
// report (t.iss.one), infrastructure paragraph: long sequences split across devices, only
// the fixed-size recurrent state exchanged).  This kernel applies one such map; fp32.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kComposeThreads = 256;
constexpr int kCols = 32;   // state columns per CTA

template <int DK>
__global__ void __launch_bounds__(kComposeThreads)
kda_state_compose_kernel(const float* __restrict__ M, const float* S, const float* N, float* out, int dv) {
    constexpr int TPR = kComposeThreads / DK;   // threads per output row (2 or 4)
    constexpr int CPT = kCols / TPR;            // columns per thread (16 or 8)
    __shared__ float ss[DK][kCols + 1];         // S[:, slice] (padded against bank conflicts)
    const int nslice = dv / kCols;
    const int slice = blockIdx.x % nslice;
    const size_t hd = blockIdx.x / nslice;
    const int c0 = kCols * slice;
    const float* Sh = S + hd * DK * dv;
    // the whole slice is read before anything is written, so out may be S itself
    for (int idx = threadIdx.x; idx < DK * kCols; idx += kComposeThreads) {
        const int k = idx / kCols, c = idx % kCols;
        ss[k][c] = Sh[(size_t)k * dv + c0 + c];
    }
    __syncthreads();
    const int i = threadIdx.x / TPR, cb = (threadIdx.x % TPR) * CPT;
    const size_t orow = (hd * DK + i) * dv + c0 + cb;
    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = N ? N[orow + j] : 0.f;
    const float* Mi = M + (hd * DK + i) * DK;
#pragma unroll 4
    for (int k = 0; k < DK; ++k) {
        const float m = __ldg(Mi + k);
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = fmaf(m, ss[k][cb + j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) out[orow + j] = acc[j];
}

}  // namespace

cudaError_t launch_state_compose(const float* M, const float* S, const float* N, float* out, int count, int dk,
                                 int dv, cudaStream_t s) {
    const unsigned grid = (unsigned)((size_t)count * (dv / kCols));
    if (dk == 128) kda_state_compose_kernel<128><<<grid, kComposeThreads, 0, s>>>(M, S, N, out, dv);
    else kda_state_compose_kernel<64><<<grid, kComposeThreads, 0, s>>>(M, S, N, out, dv);
    return cudaGetLastError();
}

}  // namespace kda
