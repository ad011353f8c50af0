// Output correction of a sequence segment that was run from a zero state: o_t += S_in^T C_t.
//
// Over a segment the state after token t is affine in the segment's start state S_in:
// S_t = Phi_t S_in + S_t^0, with Phi_t = prod_{u<=t} (I - beta_u k_u k_u^T) Diag(exp g_u) and
// S_t^0 the state from a zero start.  The read-out o_t = S_t^T q_t is therefore
// o_t^0 + S_in^T (Phi_t^T q_t): the zero-start output plus a term that needs only the
// fixed-size S_in and the per-token vector C_t = Phi_t^T q_t.  C_t is exactly the output of
// the same prefill run with v = 0 and S0 = I (its state is Phi_t, and it reads Phi_t^T q_t),
// whose final state is the segment's map M.  So a segment can be run before the state it
// starts from is known, and corrected once it arrives: the exchange of KDA context
// parallelism, which splits a long sequence over devices and passes on only the fixed-size
// state (channel post on the K3 report (t.iss.one), infrastructure paragraph).
//
// For bf16 with dk = dv = 128 the product runs on the tensor core.  A CTA takes one head and a run
// of up to 16 tiles of 128 tokens: S_in rounded to bf16 once into an MN-major tile, then per tile C
// by TMA into a 128-byte-swizzled K-major tile, D = C S_in (128 x 128 fp32) in tensor memory, and
// o_in (TMA) + D rounded to bf16 and stored by TMA.  The next tile's C is loaded as soon as the
// product has read the current one, the next o_in as soon as the store has read its staging tile,
// so the loads of one tile overlap the work on the previous one.  Other dtypes and head sizes take
// a CUDA-core kernel in fp32.
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kTok = 128;                 // tokens per tile (the tensor-core product's M)
constexpr int kD = 128;
constexpr int kTilesPerCta = 16;          // tiles of one head per CTA (S_in converted once for them)
constexpr int kThreads = 128;             // 4 warps: one TMEM lane quarter each
constexpr int kLoader = 0;                // issues the C loads and the products
constexpr int kStorer = 32;               // stores O and loads the next o_in
constexpr uint32_t OFF_C = 0;             // C tile: 2 atoms of [128 tokens][64 channels] bf16
constexpr uint32_t OFF_S = 32768;         // S_in bf16, MN-major (K = dk rows), 2 atoms
constexpr uint32_t OFF_O = 65536;         // o_in, then o_out: 2 atoms of [128 tokens][64 columns]
constexpr uint32_t SMEM_DYN = 98304 + 1024;
constexpr uint32_t ID_CS = idesc_bf16_f32(128, 128, false, true);

__global__ void __launch_bounds__(kThreads)
kda_output_correct_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_oi,
                             const __grid_constant__ CUtensorMap tm_oo, const float* S, int H, int ntiles,
                             int nsplit, int* status, unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    const uint32_t sb = smem_u32(sm);
    __shared__ uint64_t bar_c, bar_o, bar_mma, bar_drain;
    __shared__ uint32_t tmem_base_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = blockIdx.x / nsplit;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int tile0 = (int)(blockIdx.x % nsplit) * kTilesPerCta;
    const int tile1 = min(tile0 + kTilesPerCta, ntiles);

    if (tid == 0) {
        mbar_init(&bar_c, 1);
        mbar_init(&bar_o, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_drain, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_c); prefetch_tensormap(&tm_oi); prefetch_tensormap(&tm_oo);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_s, kD);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = tmem_base_s;
    auto load_c = [&](int tile) {
        mbar_arrive_expect_tx(&bar_c, 2u * 16384u);
#pragma unroll
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + OFF_C + x * 16384, &tm_c, &bar_c, 64 * x, h, tile * kTok, b);
    };
    auto load_o = [&](int tile) {
        mbar_arrive_expect_tx(&bar_o, 2u * 16384u);
#pragma unroll
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + OFF_O + x * 16384, &tm_oi, &bar_o, 64 * x, h, tile * kTok, b);
    };
    int pending_c = -1, pending_o = -1;   // iteration whose load is in flight (loader / storer)
    if (tid == kLoader) { load_c(tile0); pending_c = 0; }
    if (tid == kStorer) { load_o(tile0); pending_o = 0; }
    // S_in -> bf16 B operand (row i = dk index, columns = dv): thread i converts row i
    {
        const float4* src = reinterpret_cast<const float4*>(S + (bh * kD + tid) * kD);
#pragma unroll
        for (int j = 0; j < kD; j += 8) {
            const float4 x0 = src[j / 4], x1 = src[j / 4 + 1];
            __nv_bfloat162 p0 = __floats2bfloat162_rn(x0.x, x0.y), p1 = __floats2bfloat162_rn(x0.z, x0.w);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(x1.x, x1.y), p3 = __floats2bfloat162_rn(x1.z, x1.w);
            *reinterpret_cast<uint4*>(sm + OFF_S + sw128_offset(tid, j, 16384)) =
                make_uint4(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1),
                           *reinterpret_cast<uint32_t*>(&p2), *reinterpret_cast<uint32_t*>(&p3));
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    bool ok = true;
    for (int it = 0, tile = tile0; tile < tile1; ++it, ++tile) {
        const uint32_t par = (uint32_t)(it & 1);
        // D = C S_in, then the next C into the tile the product has read
        if (tid == kLoader) {
            ok = mbar_wait(&bar_c, par, timeout_ns);
            if (ok) {
                pending_c = -1;
                tc_fence_after_sync();
                issue_mma<8, false, 16384, true, 16384>(tbase, sb + OFF_C, sb + OFF_S, ID_CS, false);
                mma_commit(&bar_mma);
            }
        }
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        ok = mbar_wait(&bar_mma, par, timeout_ns);
        if (ok && tid == kLoader && tile + 1 < tile1) { load_c(tile + 1); pending_c = it + 1; }
        if (ok) ok = mbar_wait(&bar_o, par, timeout_ns);
        if (ok && tid == kStorer) pending_o = -1;
        ok = __syncthreads_and(ok) != 0;   // block-uniform: the TMEM loads below are warp-collective
        if (!ok) break;
        tc_fence_after_sync();
        {
            // token row r = this thread's TMEM lane: o = o_in + D, 32 columns at a time
            const int r = 32 * warp + lane;
            const uint32_t tl = tbase + ((uint32_t)(32 * warp) << 16);
#pragma unroll
            for (int cb = 0; cb < kD; cb += 32) {
                float d[32];
                tmem_ld16(tl + cb, d);
                tmem_ld16(tl + cb + 16, d + 16);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint8_t* p = sm + OFF_O + sw128_offset(r, cb + j, 16384);
                    const uint4 w = *reinterpret_cast<const uint4*>(p);
                    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&w);
                    uint32_t out[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 f = __bfloat1622float2(o2[m]);
                        __nv_bfloat162 q = __floats2bfloat162_rn(f.x + d[j + 2 * m], f.y + d[j + 2 * m + 1]);
                        out[m] = *reinterpret_cast<uint32_t*>(&q);
                    }
                    *reinterpret_cast<uint4*>(p) = make_uint4(out[0], out[1], out[2], out[3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();   // the next product overwrites D
        __syncthreads();
        if (tid == kStorer) {
            // rows past T are clipped by the tensor map; the next o_in lands once the staging tile is read
            tma_store_4d(&tm_oo, sm + OFF_O, 0, h, tile * kTok, b);
            tma_store_4d(&tm_oo, sm + OFF_O + 16384, 64, h, tile * kTok, b);
            bulk_commit_group();
            if (tile + 1 < tile1) {
                bulk_wait_read_all();
                load_o(tile + 1);
                pending_o = it + 1;
            }
        }
    }
    if (!ok && tid == 0) report_status(status, KDA_ERR_TIMEOUT);
    // nothing of this CTA may still be in flight when it exits
    if (tid == kLoader) {
        mma_commit(&bar_drain);
        if (!mbar_wait(&bar_drain, 0, timeout_ns)) report_status(status, KDA_ERR_TIMEOUT);
        if (pending_c >= 0) (void)mbar_wait(&bar_c, (uint32_t)(pending_c & 1), timeout_ns);
    }
    if (tid == kStorer) {
        bulk_wait_all();
        if (pending_o >= 0) (void)mbar_wait(&bar_o, (uint32_t)(pending_o & 1), timeout_ns);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, kD);
}

// Other dtypes and head sizes: fp32 on CUDA cores.  Per CTA one head and 16 tokens; C of those
// tokens in shared memory, S read from L2 (each column by consecutive threads).
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256)
kda_output_correct_simt_kernel(const T* C, const float* S, const T* o_in, T* o_out, int Tn, int H, int ntiles) {
    constexpr int TOK = 16;
    __shared__ float cs[TOK][DK];
    const int tile = blockIdx.x % ntiles;
    const size_t bh = blockIdx.x / ntiles;
    const size_t b = bh / H, h = bh % H;
    const int t0 = tile * TOK;
    for (int idx = threadIdx.x; idx < TOK * DK; idx += blockDim.x) {
        const int tt = idx / DK, i = idx % DK;
        const int t = t0 + tt;
        cs[tt][i] = t < Tn ? load_elem(C, ((b * Tn + t) * H + h) * DK + i) : 0.f;
    }
    __syncthreads();
    const float* Sh = S + bh * DK * DV;
    for (int idx = threadIdx.x; idx < TOK * DV; idx += blockDim.x) {
        const int tt = idx / DV, j = idx % DV;
        const int t = t0 + tt;
        if (t >= Tn) continue;
        const size_t oi = ((b * Tn + t) * H + h) * DV + j;
        float acc = load_elem(o_in, oi);
#pragma unroll 8
        for (int i = 0; i < DK; ++i) acc = fmaf(__ldg(Sh + i * DV + j), cs[tt][i], acc);
        store_elem(o_out, oi, acc);
    }
}

bool make_map128(CUtensorMap* m, const void* ptr, int B, int T, int H) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)T * H * kD * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kTok, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t launch_simt(const void* C, const float* S, const void* o_in, void* o_out, int B, int Tn, int H, int dk,
                        int dv, cudaStream_t s) {
    const int ntiles = (Tn + 15) / 16;
    const unsigned grid = (unsigned)((size_t)B * H * ntiles);
    const T* c = static_cast<const T*>(C);
    const T* oi = static_cast<const T*>(o_in);
    T* oo = static_cast<T*>(o_out);
    if (dk == 128 && dv == 128) kda_output_correct_simt_kernel<T, 128, 128><<<grid, 256, 0, s>>>(c, S, oi, oo, Tn, H, ntiles);
    else if (dk == 128) kda_output_correct_simt_kernel<T, 128, 64><<<grid, 256, 0, s>>>(c, S, oi, oo, Tn, H, ntiles);
    else if (dv == 128) kda_output_correct_simt_kernel<T, 64, 128><<<grid, 256, 0, s>>>(c, S, oi, oo, Tn, H, ntiles);
    else kda_output_correct_simt_kernel<T, 64, 64><<<grid, 256, 0, s>>>(c, S, oi, oo, Tn, H, ntiles);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_output_correct(const void* C, const float* S, const void* o_in, void* o_out, int B, int T, int H,
                                  int dk, int dv, int dtype, int* status, unsigned long long timeout_ns,
                                  cudaStream_t s) {
    if (dtype == KDA_DTYPE_BF16 && dk == kD && dv == kD) {
        static bool attr_set[64] = {false};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 64 && !attr_set[dev]) {
            e = cudaFuncSetAttribute(kda_output_correct_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SMEM_DYN);
            if (e != cudaSuccess) return e;
            attr_set[dev] = true;
        }
        CUtensorMap mc, mi, mo;
        if (!make_map128(&mc, C, B, T, H) || !make_map128(&mi, o_in, B, T, H) || !make_map128(&mo, o_out, B, T, H))
            return cudaErrorInvalidValue;
        const int ntiles = (T + kTok - 1) / kTok;
        const int nsplit = (ntiles + kTilesPerCta - 1) / kTilesPerCta;
        const unsigned grid = (unsigned)((size_t)B * H * nsplit);
        kda_output_correct_tc_kernel<<<grid, kThreads, SMEM_DYN, s>>>(mc, mi, mo, S, H, ntiles, nsplit, status,
                                                                       timeout_ns);
        return cudaGetLastError();
    }
    if (dtype == KDA_DTYPE_BF16) return launch_simt<__nv_bfloat16>(C, S, o_in, o_out, B, T, H, dk, dv, s);
    return launch_simt<float>(C, S, o_in, o_out, B, T, H, dk, dv, s);
}

}  // namespace kda
