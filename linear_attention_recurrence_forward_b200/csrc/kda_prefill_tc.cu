// KDA chunked prefill on sm_100a: TMA loads, tcgen05 tensor-core products with TMEM
// accumulators, fp32 state carried across 64-token chunks.  bf16 inputs; dk and dv each 64 or
// 128, every product 128 wide (see "Head size 64" below).
//
// Method (chunk-recurrent form of the gated delta rule: podcast show-notes section 2.1,
// RetNet chunk recurrence + Gated DeltaNet gated delta rule; delta rule of the "Day 21"
// course page, quiz Q9).  For one head and a chunk of C = 64 tokens with local index r,
// state S (dk x dv) at the chunk start, Gam_r = sum_{t<=r} g_t (per channel):
//
//   Kt_r = k_r e^{Gam_r},  Qt_r = q_r e^{Gam_r},  Kb_j = k_j e^{Gam_C - Gam_j}
//   A_rj = beta_r sum_i k_r[i] k_j[i] e^{Gam_r[i]-Gam_j[i]}   (j < r)
//   P_rj =        sum_i q_r[i] k_j[i] e^{Gam_r[i]-Gam_j[i]}   (j <= r)
//   T = (I + A)^{-1} Diag(beta)           (the WY / UT transform of the delta rule)
//   U = T (V - Kt S)                       (the delta-rule residuals of the chunk)
//   O = Qt S + P U
//   S <- Diag(e^{Gam_C}) S + Kb^T U
//
// This is an exact rewrite of the token recurrence.  The pair factors e^{Gam_r-Gam_j} are
// formed as e^{Gam_r-Gam_b} e^{Gam_b-Gam_j} against a reference token b.  The chunk is two
// 32-token blocks; both the diagonal block of block 1 and the block-1 x block-0 rectangle
// use b = 48, the diagonal block of block 0 uses b = 16.  Row-side factors are at most
// e^{5*16} = e^{80} < FLT_MAX because the log-decay is bounded below by -5 (the skill card's
// quick facts: the bounded scaled-sigmoid gate is what lets the diagonal tiles run as dense
// tensor-core matmuls).  On the rectangle a column factor e^{Gam_48-Gam_j} can underflow;
// the pair factor it belongs to is then below e^{-7.3} and the term is dropped (measured in
// fp64: at most 4.3e-4 relative to max|o| under adversarial decay, zero on the recipe inputs).
//
// CTA organisation: one (b, h) per CTA, 16 warps, two warp-specialised groups coupled by
// mbarriers so that the state-independent work of chunk c+1 overlaps the recurrence of
// chunk c:
//   prep warps 0..7    per chunk: Gam as an fp32 running sum in registers (the next chunk's g
//                      is loaded as soon as it has been read) -> per-channel constants ->
//                      bf16 operand tiles -> MMA1 (A and P in one product) -> the triangular
//                      solve on warp-level bf16 MMA tiles (diagonal blocks by a doubling
//                      product, off-diagonal blocks by a walk down each block column) ->
//                      T, P, Kb tiles.
//   serial warps 8..15 per chunk: MMA3 [Qt;Kt] S -> Y = V - Kt S -> MMA4 U = T Y ->
//                      MMA5 O = Qt S + P U, MMA6 S += Kb^T U (state decayed in TMEM first)
//                      -> O to global, S to bf16 for the next chunk.  One thread issues the
//                      products, another the O store and the v loads.
// All tcgen05 products are M = 128: products with 64 meaningful rows read 64 further rows
// of other valid shared memory into TMEM lanes that are never read.
//
// Head size 64.  The kernel always works on 128 key channels and 128 value columns.  The tensor
// maps of q, k, g (and v, o) are declared with the true channel count, so the TMA box of
// channels 64-127 of a 64-wide tensor lies wholly outside it and lands as zeros.  That is an
// exact embedding of the smaller problem: a key channel with k = q = 0 and g = 0 (or any bounded
// decay) leaves its state row at zero and adds nothing to A, P or O; a value column with v = 0
// leaves its state column, Y, U and O column at zero.  Only the state's row and column strides,
// and the O store of columns 64-127, depend on dk and dv.
#include <cudaTypedefs.h>
#include <mutex>

#include "kda_internal.cuh"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kC = 64;          // chunk length
constexpr int kD = 128;         // key channels and value columns the kernel works on (dk, dv <= kD)
constexpr int kThreads = 512;   // 16 warps
constexpr int kPrepThreads = 256;
constexpr int kSerialThreads = 256;
constexpr uint32_t kBarPrep = 1, kBarSerial = 2;   // named hardware barriers
constexpr int kIssuer = 0;                         // prep thread that issues the g loads (with the prologue chunk 0's
                                                   // only), chunk 0's q, k, and the hand-off signals
constexpr int kMma1Issuer = 224;                   // prep thread that issues MMA1 (warp 7: lightest in the solve)
constexpr int kGateWarp0 = 10, kGateWarps = 6;     // with the prologue: the recurrence warps that convert the gate

// ---- shared memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t OFF_RAW_Q = 0;           // TMA destination, bf16 [64 tok][128], 2 boxes of 8 KB
constexpr uint32_t OFF_RAW_K = 16384;
constexpr uint32_t OFF_RAW_G = 32768;
constexpr uint32_t OFF_V = 49152;           // v, then Y = V - Kt S, then U (MN-major B, K = 64 tokens)
constexpr uint32_t OFF_AP = 65536;          // prep operand region (56 KB)
constexpr uint32_t OFF_A1 = OFF_AP;                 // [Qt0;Kt0;Qt1;Kt1] block-middle refs, K-major, 2 x 16 KB
                                                    // (with the prologue, from a chunk's MMA1 to the next chunk's
                                                    // scan: that next chunk's converted gate, f16 in the g tile's layout)
constexpr uint32_t OFF_BB = OFF_AP + 32768;         // [Kh0(16);Kh1(48);Kh0(48)], K-major, 96 rows, 2 x 12 KB
// The solve's scratch, in the MMA1 B-operand space (free once MMA1 is done; the A-operand space is
// left alone): the diagonal 16x16 blocks of A in fp32 (padded rows of kLdD floats), A in bf16
// (row-major, rows of kLdA elements) for the off-diagonal blocks, and the diagonal blocks of
// X = (I+A)^-1 in bf16 (rows of kLdX elements).  bf16 rows are 16-byte aligned for ldmatrix.
constexpr int kLdD = 20, kLdA = 72, kLdX = 24;
constexpr uint32_t OFF_AFD = OFF_BB;
constexpr uint32_t OFF_AOFF = OFF_AFD + 4 * 16 * kLdD * 4;
constexpr uint32_t OFF_XD = OFF_AOFF + 64 * kLdA * 2;
constexpr uint32_t OFF_KQ = OFF_AP + 57344;          // [Qt0;Kt0;Qt1;Kt1] chunk-start ref, K-major, 2 x 16 KB
constexpr uint32_t OFF_SB = OFF_KQ + 32768;          // S in bf16, MN-major B (K = dk), 2 x 16 KB
constexpr uint32_t OFF_TP = OFF_SB + 32768;          // T and P, interleaved 4 KB pieces (16 KB)
constexpr uint32_t OFF_T = OFF_TP;                   //   T rows 0-31 at +0, rows 32-63 at +8 KB
constexpr uint32_t OFF_P = OFF_TP + 4096;            //   P rows 0-31 at +4 KB, rows 32-63 at +12 KB
constexpr uint32_t OFF_KBAR = OFF_TP + 16384;        // Kb, MN-major A (M = dk), 2 x 8 KB
constexpr uint32_t SMEM_BYTES = OFF_KBAR + 16384;    // 221184
constexpr uint32_t SMEM_DYN = SMEM_BYTES + 1024;     // + alignment slack
static_assert(OFF_XD + 4 * 16 * kLdX * 2 <= OFF_BB + 2 * 12288, "solve scratch leaves the MMA1 B space");
static_assert(OFF_BB + 2 * 12288 <= OFF_KQ, "BB overlaps KQ");

// ---- TMEM columns (fp32 accumulators, 128 lanes) ----
constexpr uint32_t TM_S = 0;     // S (dk lanes x dv columns), fp32 master state
constexpr uint32_t TM_C = 128;   // MMA3: lanes 0-31 Qt0 S, 32-63 Kt0 S, 64-95 Qt1 S, 96-127 Kt1 S; + P U
constexpr uint32_t TM_U = 256;   // MMA4: U at lanes 0-31 (tokens 0-31) and 64-95 (tokens 32-63)
constexpr uint32_t TM_P = 384;   // prep: MMA1 (96 columns)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_MMA1 = idesc_bf16_f32(128, 96, false, false);
constexpr uint32_t ID_KxMN = idesc_bf16_f32(128, 128, false, true);
constexpr uint32_t ID_MNxMN = idesc_bf16_f32(128, 128, true, true);
constexpr float kLog2e = 1.4426950408889634f;

struct TcParams {
    const __nv_bfloat16* beta;
    const float* S0;
    __nv_bfloat16* o;               // for the per-row stores of a packed sequence's partial last chunk
    float* ST;
    int* status;
    unsigned long long timeout_ns;  // limit of every mbarrier wait
    int skip_handoff;               // test hook: never signal the first KQ hand-off
    float* S_mid;                   // state after every `interval` tokens, or null
    int interval, n_mid;
    const int* cu_seqlens;          // packed sequences (B sequences over T tokens), or null
    int B, T, H;
    int dk, dv;                     // 64 or 128 each: the state's row / column counts in memory
};

// Element-wise bf16x2 product, rounded to nearest even.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) { return pack_bf16x2(v.x, v.y); }
// Two fp32 lanes in one instruction (sm_100 f32x2 arithmetic; each lane is rounded as the
// scalar operation rounds it, so results are those of the scalar code)
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Warp-level bf16 tensor-core tile D(16x8) += A(16x16, row-major) * B(16x8, column-major), fp32
// accumulate.  Fragment ownership (lane = 4*g + t): A {(g,2t..2t+1), (g+8,2t..), (g,2t+8..), (g+8,2t+8..)},
// B {(2t..2t+1, g), (2t+8.., g)}, D {(g,2t), (g,2t+1), (g+8,2t), (g+8,2t+1)}.
__device__ __forceinline__ void mma_16816(float d[4], const uint32_t a[4], const uint32_t b[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// 8x8 transpose of b16 pairs across the warp (thread i holds row i/4, columns 2(i%4) and 2(i%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// A 16x16 fp32 tile held as two m16n8 accumulator tiles d[nt] (columns 8nt..8nt+7) ...
// ... as the A operand (16x16, K = columns), rounded to bf16
__device__ __forceinline__ void afrag_of_acc(const float d[2][4], uint32_t a[4]) {
    a[0] = pack_bf16x2(d[0][0], d[0][1]); a[1] = pack_bf16x2(d[0][2], d[0][3]);
    a[2] = pack_bf16x2(d[1][0], d[1][1]); a[3] = pack_bf16x2(d[1][2], d[1][3]);
}
// ... as the B operand (K = rows) of output columns 8nt..8nt+7, rounded to bf16
__device__ __forceinline__ void bfrag_of_acc(const float d[2][4], int nt, uint32_t b[2]) {
    b[0] = movmatrix_trans(pack_bf16x2(d[nt][0], d[nt][1]));
    b[1] = movmatrix_trans(pack_bf16x2(d[nt][2], d[nt][3]));
}
// out = (acc ? out : 0) + X Y for 16x16 tiles held as accumulators (bf16 operands, fp32 sums)
__device__ __forceinline__ void mm16_acc(float out[2][4], const uint32_t ax[4], const float y[2][4], bool acc) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        uint32_t b[2];
        bfrag_of_acc(y, nt, b);
        if (!acc) out[nt][0] = out[nt][1] = out[nt][2] = out[nt][3] = 0.f;
        mma_16816(out[nt], ax, b);
    }
}

__device__ __forceinline__ float ex2_approx(float x);
// The gate prologue: beta = sigmoid(z) and the bounded log-decay g = -5 sigmoid(z) (the scaled
// sigmoid with lower bound -5 of the skill card's quick facts).  1 + e^{-z} overflows to inf for
// z << 0, which gives 0 (no decay / no write), the limit.
__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.f, 1.f + ex2_approx(-z * 1.4426950408889634f)); }
// The log-decay g = -5 sigmoid(z) of a pair of logits, scaled by 2^11 and rounded to an f16 pair.
// The prologue converts each chunk's gate logits in place to this form ahead of the scan.  The
// relative error is at most 2^-11; the scale keeps every |g| >= 2^-25 a normal f16 (below that the
// absolute error is under 2^-36), and 5 * 2^11 stays under the f16 maximum.
__device__ __forceinline__ uint32_t gate_f16x2_from_logits(uint32_t zz) {
    const float z0 = __uint_as_float(zz << 16), z1 = __uint_as_float(zz & 0xFFFF0000u);
    const float g0 = __fdividef(-5.f * 2048.f, 1.f + ex2_approx(-z0 * 1.4426950408889634f));
    const float g1 = __fdividef(-5.f * 2048.f, 1.f + ex2_approx(-z1 * 1.4426950408889634f));
    uint32_t h;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(g1), "f"(g0));
    return h;
}
__device__ __forceinline__ float2 f32x2_from_f16x2(uint32_t h) {
    float lo, hi;
    asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h));
    return make_float2(lo, hi);
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Same without flushing subnormal results (used for per-channel constants that multiply large factors).
__device__ __forceinline__ float ex2_approx_sub(float x) {
    float y;
    asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Load 64 TMEM columns of this warp's lanes (one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* r) {
#pragma unroll
    for (int cb = 0; cb < 64; cb += 16) tmem_ld16(taddr + cb, r + cb);
    tmem_wait_ld();
}

__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

// Row of the T and P tiles that holds matrix row r (0..63): rows 0-31 stay, rows 32-63 move to
// 64-95, so that the products land in the TMEM lanes of the Qt rows.
__device__ __forceinline__ int tp_row(int r) { return r < 32 ? r : r + 32; }

// Fragments from bf16 tiles in shared memory (row addresses 16-byte aligned): the A fragment of a
// 16x16 row-major block, and the B fragment of a 16x8 (K x N) block of a row-major (K rows) matrix.
__device__ __forceinline__ void ldsm_a16(uint32_t base, uint32_t row_bytes, int lane, uint32_t a[4]) {
    const uint32_t m = lane >> 3, rr = lane & 7;
    const uint32_t addr = base + (rr + 8 * (m & 1)) * row_bytes + 16 * (m >> 1);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_b16x8_trans(uint32_t base, uint32_t row_bytes, int lane, uint32_t b[2]) {
    const uint32_t rr = lane & 15;   // lanes 16-31 repeat 0-15 (their addresses are not used)
    const uint32_t addr = base + rr * row_bytes;
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(b[0]), "=r"(b[1]) : "r"(addr) : "memory");
}


// One warp's walk down block column J of X = (I + A)^-1 (its 8 output columns nt), on warp-level
// bf16 tensor-core tiles with fp32 sums.  With At_RL = X_RR A_RL (R > L >= J; independent products,
// formed first), X_RJ = -sum_{L=J}^{R-1} At_RL X_LJ for R = J+1 .. 3, so the dependent chain is one
// accumulation per block.  Each X_LJ it needs is the diagonal block (level 0's transposed copy) or
// one it has just formed, kept as a B fragment in registers: no other warp is waited for.  T =
// X Diag(beta) entries are written as they are formed, row r times rowf[r] when rowf is given.
// (bf16 operands at these points leave the output error unchanged in the chunk model.)
template <int J>
__device__ __forceinline__ void offdiag_column(uint32_t sb, const float* beta, const float* rowf, uint8_t* sm, int nt,
                                               int lane) {
    constexpr int NR = 3 - J;   // blocks below the diagonal in this column
    const int g4 = lane >> 2, t4 = lane & 3;
    uint32_t at[NR][NR][4];     // A fragments of At_RL, [R - J - 1][L - J]
#pragma unroll
    for (int R = J + 1; R < 4; ++R) {
        uint32_t xr[4];
        ldsm_a16(sb + OFF_XD + 16 * R * kLdX * 2, kLdX * 2, lane, xr);
#pragma unroll
        for (int L = J; L < R; ++L) {
            float d[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                uint32_t bf[2];
                ldsm_b16x8_trans(sb + OFF_AOFF + (16 * R) * kLdA * 2 + (16 * L + 8 * n) * 2, kLdA * 2, lane, bf);
                d[n][0] = d[n][1] = d[n][2] = d[n][3] = 0.f;
                mma_16816(d[n], xr, bf);
            }
            afrag_of_acc(d, at[R - J - 1][L - J]);
        }
    }
    uint32_t xb[NR][2];         // B fragments of X_LJ, L = J .. 2
    ldsm_b16x8_trans(sb + OFF_XD + 16 * J * kLdX * 2 + 8 * nt * 2, kLdX * 2, lane, xb[0]);
    const int col = 16 * J + 8 * nt + 2 * t4;
    const float b0 = beta[col], b1 = beta[col + 1];
#pragma unroll
    for (int R = J + 1; R < 4; ++R) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int L = J; L < R; ++L) mma_16816(x, at[R - J - 1][L - J], xb[L - J]);
        float2 t0v = mul2(make_float2(-x[0], -x[1]), make_float2(b0, b1));
        float2 t1v = mul2(make_float2(-x[2], -x[3]), make_float2(b0, b1));
        if (rowf) {
            const float f0 = rowf[16 * R + g4], f1 = rowf[16 * R + g4 + 8];
            t0v = mul2(t0v, make_float2(f0, f0));
            t1v = mul2(t1v, make_float2(f1, f1));
        }
        *reinterpret_cast<uint32_t*>(sm + OFF_T + sw128_offset(tp_row(16 * R + g4), col, 8192)) = pack_bf16x2(t0v);
        *reinterpret_cast<uint32_t*>(sm + OFF_T + sw128_offset(tp_row(16 * R + g4 + 8), col, 8192)) = pack_bf16x2(t1v);
        if (R < 3) {
            xb[R - J][0] = movmatrix_trans(pack_bf16x2(-x[0], -x[1]));
            xb[R - J][1] = movmatrix_trans(pack_bf16x2(-x[2], -x[3]));
        }
    }
}

// kFused: the gate and normalisation prologue (q, k raw; g, beta as logits).  Its extra work is kept
// off the prep group's path where it can be: six recurrence warps convert the gate logits to log-decays
// two chunks ahead, while they would otherwise wait for the next MMA3; the operand tiles are those of
// the raw q, k, and the row norms (one pass after the tiles) are applied where elements are scaled
// anyway.  kPacked: packed variable-length sequences.  Compiled separately so that the plain path
// carries neither.
template <bool kFused, bool kPacked>
__global__ void __launch_bounds__(kThreads, 1)
kda_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    // Align to 1024 B (the swizzle atoms need it) by offsetting the shared array itself, so the
    // compiler keeps every access in the shared state space.
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    const uint32_t sb = smem_u32(sm);

    // TMA / MMA completion barriers (one phase per chunk) and prep -> serial hand-offs.
    __shared__ uint64_t bar_qk, bar_g, bar_v, bar_ap, bar_c, bar_u, bar_os, bar_kq, bar_tpk;
    __shared__ uint64_t bar_drain_p, bar_drain_s, bar_drain_g;
    __shared__ uint64_t bar_gc;   // with the prologue: a chunk's gate converted (one arrival per converting warp)
    __shared__ uint32_t tmem_base_s;
    __shared__ __align__(16) float s_beta[kC];
    __shared__ __align__(16) float s_gamma[2][kD];     // e^{Gam_63} per channel, by chunk parity (float2 stores)
    __shared__ __align__(16) float s_qsum[4][kD];      // g summed over each 16-token quarter
    __shared__ __align__(16) float s_g1648[2][kD];     // g of tokens 16 and 48 (raw g is dead after the scan)
    __shared__ __align__(16) float s_norm[2][2 * kC];  // with the prologue: 1/|q_t|, then 1/|k_t|, by chunk parity

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto tid_is_zero = [&]() { return tid == 0; };
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const bool is_prep = warp < 8;
    const int colhalf = (warp >> 2) & 1;       // which 64 columns of a 128-wide result (per group)
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    // This CTA's tokens: rows tok0 .. tok0 + T - 1 of batch entry bmap of the tensor maps, i.e.
    // [B, T, H, d] as laid out, or sequence b of packed sequences (maps with one batch entry of
    // all tokens; offsets from cu_seqlens, checked here as a whole: offsets that are not one
    // valid, non-overlapping layout are reported and every sequence is processed as empty)
    int tok0 = 0, bmap = b, T = p.T;
    if (kPacked) {
        const bool valid = packed_offsets_valid(p.cu_seqlens, p.B, p.T);
        if (!valid && tid_is_zero()) report_status(p.status, KDA_ERR_INVALID_ARG);
        tok0 = valid ? p.cu_seqlens[b] : 0;
        bmap = 0;
        T = valid ? p.cu_seqlens[b + 1] - tok0 : 0;
    }
    const size_t row0 = (size_t)bmap * p.T + tok0;   // token-axis row of this CTA's first token
    const int nchunks = (T + kC - 1) / kC;

    if (tid == 0) {
        mbar_init(&bar_qk, 1); mbar_init(&bar_g, 1); mbar_init(&bar_v, 1); mbar_init(&bar_ap, 1);
        mbar_init(&bar_c, 1); mbar_init(&bar_u, 1); mbar_init(&bar_os, 1); mbar_init(&bar_kq, 1);
        mbar_init(&bar_tpk, 1); mbar_init(&bar_drain_p, 1); mbar_init(&bar_drain_s, 1); mbar_init(&bar_drain_g, 1);
        mbar_init(&bar_gc, kGateWarps);
        fence_mbar_init();
        prefetch_tensormap(&tm_q); prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_g); prefetch_tensormap(&tm_v); prefetch_tensormap(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_s, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = tmem_base_s;
    const uint32_t tlane = tbase + ((uint32_t)(32 * quarter) << 16);  // this warp's lane quarter

    // raw q and k are read until the chunk's operand tiles are written; raw g only by the scan,
    // so the next chunk's g is loaded a step earlier than its q and k
    auto load_qk = [&](int chunk) {
        mbar_arrive_expect_tx(&bar_qk, 2u * 16384u);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + OFF_RAW_Q + x * 8192, &tm_q, &bar_qk, 64 * x, h, tok0 + chunk * kC, bmap);
            tma_load_4d(sm + OFF_RAW_K + x * 8192, &tm_k, &bar_qk, 64 * x, h, tok0 + chunk * kC, bmap);
        }
    };
    auto load_g = [&](int chunk) {
        mbar_arrive_expect_tx(&bar_g, 16384u);
#pragma unroll
        for (int x = 0; x < 2; ++x)
            tma_load_4d(sm + OFF_RAW_G + x * 8192, &tm_g, &bar_g, 64 * x, h, tok0 + chunk * kC, bmap);
    };
    auto load_v = [&](int chunk) {
        mbar_arrive_expect_tx(&bar_v, 16384u);
#pragma unroll
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + OFF_V + x * 8192, &tm_v, &bar_v, 64 * x, h, tok0 + chunk * kC, bmap);
    };

    bool ok = true;
    if (is_prep) {
        // ====================================================================== prep group
        const int ptid = tid;                               // 0..255
        int pending_g = -1, pending_qk = -1;                // chunks whose g / q,k loads this issuer has in flight
        if (ptid == kIssuer) { load_g(0); load_qk(0); pending_g = 0; pending_qk = 0; }
        // T's strictly upper 16x16 blocks stay zero for the whole sequence: clear the tile once
        for (int idx = ptid; idx < 512; idx += kPrepThreads)
            *reinterpret_cast<uint4*>(sm + OFF_T + sw128_offset(tp_row(idx >> 3), (idx & 7) * 8, 8192)) =
                make_uint4(0u, 0u, 0u, 0u);
        float* AFD = reinterpret_cast<float*>(sm + OFF_AFD);
        // this thread's part of the Gam scan and of the element-wise step: channels ch0, ch0 + 1 of the
        // 16 tokens of quarter tq (a warp covers 64 channels of one quarter)
        const int tq = warp >> 1;
        const int hq = tq >> 1;                              // 32-token block (reference token 16 or 48)
        const int ch0 = 64 * (warp & 1) + 2 * lane;
        // beta of the next chunk, loaded a chunk ahead as raw bf16 bits (converted only when it is
        // stored, so the load's latency is never waited for)
        const unsigned short* beta_bits = reinterpret_cast<const unsigned short*>(p.beta);
        auto fetch_beta = [&](int chunk) -> unsigned short {
            const int t = chunk * kC + ptid;
            return (ptid < kC && t < T) ? beta_bits[(row0 + t) * p.H + h] : (unsigned short)0;
        };
        unsigned short beta_next = fetch_beta(0);
        for (int chunk = 0; chunk < nchunks; ++chunk) {
            const uint32_t par = chunk & 1, ppar = par ^ 1u;
            // ---- P1: beta; this chunk's g
            if (ptid < kC) {
                const float bz = __uint_as_float((uint32_t)beta_next << 16);
                // with the prologue beta is a logit; a padding token keeps beta = 0
                s_beta[ptid] = kFused ? (chunk * kC + ptid < T ? sigmoid_fast(bz) : 0.f) : bz;
            }
            if (chunk + 1 < nchunks) beta_next = fetch_beta(chunk + 1);
            // every thread: its own view of the TMA data (with the prologue: of the converted gate,
            // which recurrence warps write into the MMA1 A space from the TMA data)
            ok = mbar_wait(kFused ? &bar_gc : &bar_g, par, p.timeout_ns);
            if (ok && ptid == kIssuer) pending_g = -1;
            // ---- P2: Gam = in-chunk prefix sum of g in fp32: the running sum over this quarter,
            // then the totals of the quarters before it
            // rows past nvalid are padding: the tensor map reads zeros there for the [B, T, H, d] layout,
            // but the next sequence's rows for packed sequences, and a zero logit is no zero gate
            const int nvalid = min(kC, T - chunk * kC);
            float2 gam[16];
            {
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(sm + (kFused ? OFF_A1 : OFF_RAW_G) +
                                                                          sw128_offset(16 * tq + i, ch0, 8192));
                    float g0, g1;
                    if (kFused) {   // 2^11 g in f16 (exact rescaling)
                        const float2 h = f32x2_from_f16x2(w);
                        g0 = h.x * 0x1p-11f;
                        g1 = h.y * 0x1p-11f;
                    } else {
                        g0 = __uint_as_float(w << 16);
                        g1 = __uint_as_float(w & 0xFFFF0000u);
                    }
                    if ((kFused || kPacked) && 16 * tq + i >= nvalid) g0 = g1 = 0.f;
                    acc = add2(acc, make_float2(g0, g1));
                    gam[i] = acc;
                }
                *reinterpret_cast<float2*>(&s_qsum[tq][ch0]) = acc;
                if (tq & 1)   // the first token of quarter 1 (3) is token 16 (48): its sum is its g
                    *reinterpret_cast<float2*>(&s_g1648[tq >> 1][ch0]) = gam[0];
            }
            ok = named_bar_and(kBarPrep, kPrepThreads, ok);
            if (!ok) break;
            // raw g of this chunk is consumed: load the next chunk's
            // (with the prologue the recurrence warps that convert the gate load it)
            if (!kFused && ptid == kIssuer && chunk + 1 < nchunks) { load_g(chunk + 1); pending_g = chunk + 1; }
            {
                float2 carry = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int qq = 0; qq < tq; ++qq) carry = add2(carry, *reinterpret_cast<const float2*>(&s_qsum[qq][ch0]));
#pragma unroll
                for (int i = 0; i < 16; ++i) gam[i] = add2(gam[i], carry);
            }
            // the reference rows Gam_16, Gam_31, Gam_48, Gam_63 of this thread's channels, from the
            // quarter sums and g of tokens 16 and 48 (each thread forms its own: no exchange)
            float r16[2], r31[2], r48[2], r63[2];
            {
                const float2 s0 = *reinterpret_cast<const float2*>(&s_qsum[0][ch0]);
                const float2 s1 = *reinterpret_cast<const float2*>(&s_qsum[1][ch0]);
                const float2 s2 = *reinterpret_cast<const float2*>(&s_qsum[2][ch0]);
                const float2 s3 = *reinterpret_cast<const float2*>(&s_qsum[3][ch0]);
                const float2 g16v = *reinterpret_cast<const float2*>(&s_g1648[0][ch0]);
                const float2 g48v = *reinterpret_cast<const float2*>(&s_g1648[1][ch0]);
                const float2 c2 = add2(s0, s1), c3 = add2(c2, s2);
                const float2 v16 = add2(g16v, s0), v48 = add2(g48v, c3), v63 = add2(c3, s3);
                r16[0] = v16.x; r16[1] = v16.y;
                r31[0] = c2.x; r31[1] = c2.y;
                r48[0] = v48.x; r48[1] = v48.y;
                r63[0] = v63.x; r63[1] = v63.y;
            }
            if (tq == 3)   // e^{Gam_63} for the state decay
                *reinterpret_cast<float2*>(&s_gamma[par][ch0]) =
                    make_float2(ex2_approx_sub(r63[0] * kLog2e), ex2_approx_sub(r63[1] * kLog2e));
            // ---- P3: operand tiles (KQ may be rewritten once MMA3 of the previous chunk is done;
            // every thread waits for that itself, the vote is at the next barrier)
            if (ok) {
                ok = mbar_wait(&bar_qk, par, p.timeout_ns);
                if (ok && ptid == kIssuer) pending_qk = -1;
            }
            if (chunk > 0 && ok) ok = mbar_wait(&bar_c, ppar, p.timeout_ns);
            uint32_t kb[16];  // Kb of these tokens, written once the previous chunk released the tile
            {
                // per channel, against the block's reference token m: Gam_m*log2e, e^{Gam_63-Gam_m},
                // e^{Gam_m} (bf16 pair), and for block 0 the two factors of the column change to
                // token 48, e^{Gam_31-Gam_16} and e^{Gam_48-Gam_31}.  Each factor spans at most 17
                // tokens, so at g >= -5 it stays a normal float.
                float2 ngmL, ce, f1 = make_float2(0.f, 0.f), f2 = make_float2(0.f, 0.f);
                float em[2];
                {
                    const float* g16 = r16;
                    const float* g31 = r31;
                    const float* g48 = r48;
                    const float* g63 = r63;
                    float gmL[2], c[2], a[2] = {0.f, 0.f}, b[2] = {0.f, 0.f};
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float gm = hq ? g48[u] : g16[u];
                        gmL[u] = gm * kLog2e;
                        c[u] = ex2_approx_sub((g63[u] - gm) * kLog2e);
                        em[u] = ex2_approx_sub(gm * kLog2e);
                        if (hq == 0) {
                            a[u] = ex2_approx_sub((g31[u] - g16[u]) * kLog2e);
                            b[u] = ex2_approx_sub((g48[u] - g31[u]) * kLog2e);
                        }
                    }
                    ngmL = make_float2(-gmL[0], -gmL[1]);
                    ce = make_float2(c[0], c[1]);
                    f1 = make_float2(a[0], a[1]);
                    f2 = make_float2(b[0], b[1]);
                }
                const uint32_t cmb = pack_bf16x2(em[0], em[1]);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = 16 * tq + i;
                    const int rq = 64 * hq + (t & 31), rk = rq + 32;   // MMA1 rows [Qt0;Kt0;Qt1;Kt1]
                    uint32_t qw = *reinterpret_cast<const uint32_t*>(sm + OFF_RAW_Q + sw128_offset(t, ch0, 8192));
                    uint32_t kw = *reinterpret_cast<const uint32_t*>(sm + OFF_RAW_K + sw128_offset(t, ch0, 8192));
                    if (kPacked && t >= nvalid) qw = kw = 0u;
                    const float2 kv = make_float2(__uint_as_float(kw << 16), __uint_as_float(kw & 0xFFFF0000u));
                    const float2 x = fma2(gam[i], make_float2(kLog2e, kLog2e), ngmL);
                    const float2 E = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    const float2 I = make_float2(ex2_approx(-x.x), ex2_approx(-x.y));
                    const float2 kI = mul2(kv, I);
                    // MMA1 operands: A rows [Qt0;Kt0;Qt1;Kt1], B rows [Kh0(16);Kh1(48);Kh0(48)]: bf16 q (k)
                    // times the bf16-rounded factor.  With the prologue q and k are the raw rows here;
                    // their norms are applied further on (see the norm pass below)
                    const uint32_t e2 = pack_bf16x2(E), i2 = pack_bf16x2(I);
                    const uint32_t a1q = mul_bf16x2(qw, e2);
                    const uint32_t a1k = mul_bf16x2(kw, e2);
                    const uint32_t b1 = mul_bf16x2(kw, i2);
                    *reinterpret_cast<uint32_t*>(sm + OFF_A1 + sw128_offset(rq, ch0, 16384)) = a1q;
                    *reinterpret_cast<uint32_t*>(sm + OFF_A1 + sw128_offset(rk, ch0, 16384)) = a1k;
                    *reinterpret_cast<uint32_t*>(sm + OFF_BB + sw128_offset(t, ch0, 12288)) = b1;
                    // block-0 keys against token 48: k e^{Gam_16-Gam_j} e^{Gam_31-Gam_16} e^{Gam_48-Gam_31},
                    // multiplied left to right; the middle product k e^{Gam_31-Gam_j} never exceeds |k|,
                    // so a factor flushes to zero only when the exact product is below the fp32 range
                    if (hq == 0)
                        *reinterpret_cast<uint32_t*>(sm + OFF_BB + sw128_offset(64 + t, ch0, 12288)) =
                            pack_bf16x2(mul2(mul2(kI, f1), f2));
                    // MMA3 operand, the same rows against the chunk start: the bf16 tile times bf16 e^{Gam_m}
                    *reinterpret_cast<uint32_t*>(sm + OFF_KQ + sw128_offset(rq, ch0, 16384)) = mul_bf16x2(a1q, cmb);
                    *reinterpret_cast<uint32_t*>(sm + OFF_KQ + sw128_offset(rk, ch0, 16384)) = mul_bf16x2(a1k, cmb);
                    kb[i] = pack_bf16x2(mul2(kI, ce));
                }
            }
            if (kFused) {
                // 1/|x| of every raw q and k row of the chunk (row = thread/2, 64 channels per thread).
                // q and k enter every product of the chunk linearly, so their norms are applied where
                // an element is scaled anyway, not to the operand tiles: 1/|k| on A (row and column),
                // on the rows of T and on Kt S in Y; 1/|q| on O.  (With Kn = Diag(1/|k|): A' = Diag(beta)
                // Kn A Kn, U' = T' (V - Kn Kt S); MMA5 and MMA6 then take U~ = Kn U' with the raw P and Kb,
                // since P' = Diag(1/|q|) P Kn and Kb' = Kn Kb.)  This pass runs after the operand tiles,
                // off their path, and before the hand-off that lets the next q, k overwrite the raw tiles.
                const int row = ptid >> 1, half = ptid & 1, t = row & (kC - 1);
                const uint8_t* tile = sm + (row < kC ? OFF_RAW_Q : OFF_RAW_K) + half * 8192 + t * 128;
                float2 ss2 = make_float2(0.f, 0.f);   // even and odd channels
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(tile + ((j ^ (t & 7)) << 4));
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x2 = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
                        ss2 = fma2(x2, x2, ss2);
                    }
                }
                float ss = ss2.x + ss2.y;
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if (half == 0) s_norm[par][row] = ss > 0.f ? rsqrtf(ss) : 0.f;
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            ok = named_bar_and(kBarPrep, kPrepThreads, ok);
            if (!ok) break;
            // MMA1 (A and P of the chunk) straight from this group: it is on this group's path
            if (ptid == kMma1Issuer) {
                tc_fence_after_sync();
                issue_mma<8, false, 16384, false, 12288>(tbase + TM_P, sb + OFF_A1, sb + OFF_BB, ID_MMA1, false);
                mma_commit(&bar_ap);
            }
            // KQ of this chunk is ready and its raw q, k consumed: the recurrence group's leader
            // issues MMA3 and the next chunk's q, k loads
            if (ptid == kIssuer && !(p.skip_handoff && chunk == 0)) mbar_arrive(&bar_kq);
            // ---- P4: Kb tile, P and A from TMEM, triangular solve, T tile
            if (chunk > 0) ok = mbar_wait(&bar_os, ppar, p.timeout_ns);  // T, P, Kb released
            if (ok) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    *reinterpret_cast<uint32_t*>(sm + OFF_KBAR + sw128_offset(16 * tq + i, ch0, 8192)) = kb[i];
            }
            if (ok) ok = mbar_wait(&bar_ap, par, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);   // warp-uniform: the TMEM loads below are warp-collective
            tc_fence_after_sync();
            if (ok) {
                // TMEM lane L of MMA1: quarter 0 Qt0 rows, 1 Kt0 rows, 2 Qt1 rows, 3 Kt1 rows.
                // Columns of a row r: j < 32 from cols 0..31 (block 0) or 64..95 (block 1 rows);
                // j >= 32 zero (block 0) or cols 32..63 (block 1).  colhalf picks j < 32 / j >= 32.
                const bool is_q = (quarter & 1) == 0;
                const int r = 32 * (quarter >> 1) + lane;
                const int jb = 32 * colhalf;
                float row[32];
                if (quarter < 2) {
                    if (colhalf == 0) {
                        tmem_ld16(tlane + TM_P, row);
                        tmem_ld16(tlane + TM_P + 16, row + 16);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) row[j] = 0.f;
                    }
                } else {
                    const uint32_t col = colhalf == 0 ? 64u : 32u;
                    tmem_ld16(tlane + TM_P + col, row);
                    tmem_ld16(tlane + TM_P + col + 16, row + 16);
                    tmem_wait_ld();
                }
                if (is_q) {
                    // P row r: lower triangle including the diagonal
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = (jb + j + e <= r) ? row[j + e] : 0.f;
                        *reinterpret_cast<uint4*>(sm + OFF_P + sw128_offset(tp_row(r), jb + j, 8192)) = pack8(v8);
                    }
                } else {
                    // A row r: strictly lower, scaled by beta_r (select first: masked entries may be inf),
                    // in bf16; the diagonal block's 16 entries also in fp32 (quarter 1 with columns
                    // 0-31 and quarter 3 with columns 32-63 hold the diagonal blocks)
                    const float br = kFused ? s_beta[r] * s_norm[par][kC + r] : s_beta[r];
                    float w[32];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float2 pr = mul2(make_float2(row[j], row[j + 1]), make_float2(br, br));
                        if (kFused) pr = mul2(pr, *reinterpret_cast<const float2*>(&s_norm[par][kC + jb + j]));
                        w[j] = (jb + j < r) ? pr.x : 0.f;
                        w[j + 1] = (jb + j + 1 < r) ? pr.y : 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *reinterpret_cast<uint4*>(sm + OFF_AOFF + r * kLdA * 2 + (jb + j) * 2) = pack8(w + j);
                    if ((quarter == 1 && colhalf == 0) || (quarter == 3 && colhalf == 1)) {
                        const bool hi = (r & 16) != 0;    // the row's diagonal block is columns 16-31 of the 32
                        float* dst = AFD + ((r >> 4) * 16 + (r & 15)) * kLdD;
#pragma unroll
                        for (int j = 0; j < 16; j += 4)
                            *reinterpret_cast<float4*>(dst + j) = make_float4(hi ? w[16 + j] : w[j], hi ? w[17 + j] : w[j + 1],
                                                                              hi ? w[18 + j] : w[j + 2], hi ? w[19 + j] : w[j + 3]);
                    }
                }
            }
            tc_fence_before_sync();  // the next chunk's MMA1 reuses these TMEM columns
            ok = named_bar_and(kBarPrep, kPrepThreads, ok);
            if (!ok) break;
            // diagonal 16x16 blocks of X = (I + A)^-1, one warp per block: the strictly lower block N
            // is nilpotent (N^16 = 0), so (I + N)^-1 = (I - N)(I + N^2)(I + N^4)(I + N^8), formed by
            // warp-level tensor-core products (bf16 operands, fp32 sums) in four dependent rounds
            if (warp < 4) {
                const int o0 = 16 * warp, g4 = lane >> 2, t4 = lane & 3;
                float nn[2][4], xm[2][4];  // N, then N^2, N^4, N^8; the running product
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int row = g4 + 8 * hr, col = 8 * nt + 2 * t4;
                        const float2 v = *reinterpret_cast<const float2*>(AFD + (o0 + row) * kLdD + col);
                        nn[nt][2 * hr] = v.x;
                        nn[nt][2 * hr + 1] = v.y;
                        xm[nt][2 * hr] = (row == col ? 1.f : 0.f) - v.x;
                        xm[nt][2 * hr + 1] = (row == col + 1 ? 1.f : 0.f) - v.y;
                    }
#pragma unroll
                for (int round = 0; round < 3; ++round) {
                    uint32_t an[4], ax[4];
                    afrag_of_acc(nn, an);
                    float sq[2][4];
                    mm16_acc(sq, an, nn, false);        // N^(2^(round+1))
                    afrag_of_acc(xm, ax);
                    mm16_acc(xm, ax, sq, true);         // X <- X (I + N^(2^(round+1)))
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) nn[nt][e] = sq[nt][e];
                }
                // X (bf16, for the off-diagonal blocks) and T = X Diag(beta) (bf16)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = 8 * nt + 2 * t4;
                    const float b0 = s_beta[o0 + col], b1 = s_beta[o0 + col + 1];
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int row = g4 + 8 * hr;
                        const float x0 = xm[nt][2 * hr], x1 = xm[nt][2 * hr + 1];
                        *reinterpret_cast<uint32_t*>(sm + OFF_XD + ((o0 + row) * kLdX + col) * 2) = pack_bf16x2(x0, x1);
                        float2 tv = mul2(make_float2(x0, x1), make_float2(b0, b1));
                        if (kFused) { const float f = s_norm[par][kC + o0 + row]; tv = mul2(tv, make_float2(f, f)); }
                        *reinterpret_cast<uint32_t*>(sm + OFF_T + sw128_offset(tp_row(o0 + row), o0 + col, 8192)) = pack_bf16x2(tv);
                    }
                }
            }
            named_bar_sync(kBarPrep, kPrepThreads);
            // off-diagonal blocks, one block column per warp pair (8 output columns per warp)
            if (warp < 6) {
                const int nt = warp & 1;
                const float* rowf = kFused ? &s_norm[par][kC] : nullptr;
                if (warp < 2) offdiag_column<0>(sb, s_beta, rowf, sm, nt, lane);
                else if (warp < 4) offdiag_column<1>(sb, s_beta, rowf, sm, nt, lane);
                else offdiag_column<2>(sb, s_beta, rowf, sm, nt, lane);
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrep, kPrepThreads);
            if (ptid == 0) mbar_arrive(&bar_tpk);  // T, P, Kb and gamma of this chunk are ready
        }
        if (!ok && ptid == 0) report_status(p.status, KDA_ERR_TIMEOUT);
        // drain: no MMA or TMA issued by this group may still be in flight
        if (ptid == kMma1Issuer) {
            mma_commit(&bar_drain_g);
            if (!mbar_wait(&bar_drain_g, 0, p.timeout_ns)) report_status(p.status, KDA_ERR_TIMEOUT);
        }
        if (ptid == kIssuer) {
            mma_commit(&bar_drain_p);
            if (!mbar_wait(&bar_drain_p, 0, p.timeout_ns)) report_status(p.status, KDA_ERR_TIMEOUT);
            if (pending_g >= 0) (void)mbar_wait(&bar_g, (uint32_t)(pending_g & 1), p.timeout_ns);
            if (pending_qk >= 0) (void)mbar_wait(&bar_qk, (uint32_t)(pending_qk & 1), p.timeout_ns);
        }
    } else {
        // ====================================================================== serial group
        const int stid = tid - kPrepThreads;                // 0..255
        // Two single-thread roles: the leader (stid 0) issues the tensor-core products and the q, k loads;
        // the I/O thread (stid 32) stores O and loads the next v, so that the wait for the O store to
        // have read its staging tile never holds up the next chunk's MMA3.
        int pending = -1;                                   // I/O thread: chunk whose v load is in flight
        // With the prologue warps kGateWarp0.. of this group convert each chunk's gate logits (bf16 z ->
        // f16 2^11 g), two chunks ahead of the prep group's scan, in the time they otherwise wait for the
        // next chunk's MMA3.  The result goes to the MMA1 A space, free from the completion of the
        // previous chunk's MMA1 (which also means the scan and operand tiles before it are done) to
        // the next scan; the raw g buffer is then free at once and the next chunk's g is loaded.  No
        // wait here can see a phase ahead: the next g load, MMA1 and conversion all follow this one.
        int pending_g = -1;                                 // gate loader (warp kGateWarp0, lane 0)
        const bool gate_warp = kFused && warp >= kGateWarp0 && warp < kGateWarp0 + kGateWarps;
        auto convert_gate = [&](int c) -> bool {
            bool got = c == 0 || mbar_wait(&bar_ap, (uint32_t)((c - 1) & 1), p.timeout_ns);
            got = got && mbar_wait(&bar_g, (uint32_t)(c & 1), p.timeout_ns);
            if (got) {
                const uint4* src = reinterpret_cast<const uint4*>(sm + OFF_RAW_G);
                uint4* dst = reinterpret_cast<uint4*>(sm + OFF_A1);
#pragma unroll 1
                for (int idx = tid - 32 * kGateWarp0; idx < kC * kD * 2 / 16; idx += 32 * kGateWarps) {
                    const uint4 w = src[idx];
                    dst[idx] = make_uint4(gate_f16x2_from_logits(w.x), gate_f16x2_from_logits(w.y),
                                          gate_f16x2_from_logits(w.z), gate_f16x2_from_logits(w.w));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_gc);
            if (warp == kGateWarp0 && lane == 0) {
                // every converting warp has read the raw tile: the next chunk's g may land on it
                got = mbar_wait(&bar_gc, (uint32_t)(c & 1), p.timeout_ns) && got;
                if (pending_g == c) pending_g = -1;
                if (got && c + 1 < nchunks) {
                    fence_proxy_async_smem();
                    load_g(c + 1);
                    pending_g = c + 1;
                }
            }
            return got;
        };
        int pending_qk = -1;                                // leader: last chunk whose q,k loads it issued
        // Once the prep group has published chunk c's operand tiles (bar_kq): MMA3 = [Qt0;Kt0;Qt1;Kt1] S
        // and the raw q, k of chunk c+1 into the buffers the prep group has finished reading.
        auto issue_for_chunk = [&](int c) {
            tc_fence_after_sync();
            issue_mma<8, false, 16384, true, 16384>(tbase + TM_C, sb + OFF_KQ, sb + OFF_SB, ID_KxMN, false);
            mma_commit(&bar_c);
            if (c + 1 < nchunks) { load_qk(c + 1); pending_qk = c + 1; }
        };
        // initial state: fp32 into TMEM, bf16 copy into the MN-major S tile
        {
            const int i = 32 * quarter + lane;
            const int cb0 = 64 * colhalf;
            float r[64];
            if (p.S0 && i < p.dk && cb0 < p.dv) {
                const float4* src = reinterpret_cast<const float4*>(p.S0 + ((size_t)bh * p.dk + i) * p.dv + cb0);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 x = src[j];
                    r[4 * j] = x.x; r[4 * j + 1] = x.y; r[4 * j + 2] = x.z; r[4 * j + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) r[j] = 0.f;
            }
#pragma unroll
            for (int cb = 0; cb < 64; cb += 16) tmem_st16(tlane + TM_S + cb0 + cb, r + cb);
            tmem_wait_st();
#pragma unroll
            for (int j = 0; j < 64; j += 8)
                *reinterpret_cast<uint4*>(sm + OFF_SB + sw128_offset(i, cb0 + j, 16384)) = pack8(r + j);
        }
        if (stid == 32 && nchunks > 0) { load_v(0); pending = 0; }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        named_bar_sync(kBarSerial, kSerialThreads);
        // ---- S1 of chunk 0: MMA3 once the prep group has the operand tiles (later chunks issue it
        // at the end of the previous chunk)
        if (stid == 0 && nchunks > 0) {
            ok = mbar_wait(&bar_kq, 0u, p.timeout_ns);
            if (ok) issue_for_chunk(0);
        }
        if (gate_warp) {   // the gates of chunks 0 and 1 (the loop converts chunk c + 2)
            if (warp == kGateWarp0 && lane == 0 && nchunks > 0) pending_g = 0;   // loaded by the prep group
            if (nchunks > 0 && !convert_gate(0)) ok = false;
            if (nchunks > 1 && !convert_gate(1)) ok = false;
        }
        // With the prologue this group reads each chunk's norms (Y and O), which the prep group writes
        // before that chunk's KQ hand-off.  The leader waits for the hand-off (acquire) before it meets
        // the other threads at the barrier at the top of the chunk's loop iteration, and every read
        // comes after that barrier, so the norms are visible to all of them.
        for (int chunk = 0; chunk < nchunks; ++chunk) {
            const uint32_t par = chunk & 1;
            const int t0 = chunk * kC;
            // Y = V - Kt S (Kt rows sit in lanes 32-63 and 96-127), in place over v
            if (ok) ok = mbar_wait(&bar_c, par, p.timeout_ns);
            if (ok) ok = mbar_wait(&bar_v, par, p.timeout_ns);
            tc_fence_after_sync();
            ok = named_bar_and(kBarSerial, kSerialThreads, ok);
            if (!ok) break;
            if (stid == 32) pending = -1;
            if (quarter & 1) {
                const int tj = 32 * (quarter >> 1) + lane;
                float ks[64];
                tmem_ld64(tlane + TM_C + 64 * colhalf, ks);
                // with the prologue Kt S is that of the raw k row: Y = V - (Kt S) / |k|
                const float nk = kFused ? -s_norm[par][kC + tj] : -1.f;
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    const uint32_t off = sw128_offset(tj, 64 * colhalf + j, 8192);
                    const uint4 vv = *reinterpret_cast<const uint4*>(sm + OFF_V + off);
                    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vv);
                    float y[8];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 yy = kFused ? fma2(make_float2(ks[j + 2 * m], ks[j + 2 * m + 1]), make_float2(nk, nk),
                                                        __bfloat1622float2(v2[m]))
                                                 : sub2(__bfloat1622float2(v2[m]), make_float2(ks[j + 2 * m], ks[j + 2 * m + 1]));
                        y[2 * m] = yy.x;
                        y[2 * m + 1] = yy.y;
                    }
                    *reinterpret_cast<uint4*>(sm + OFF_V + off) = pack8(y);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar_sync(kBarSerial, kSerialThreads);
            // ---- S2: MMA4 U = T Y once the prep group has T, P, Kb; decay the state meanwhile
            if (stid == 0) {
                ok = mbar_wait(&bar_tpk, par, p.timeout_ns);
                if (ok) {
                    tc_fence_after_sync();
                    issue_mma<4, false, 0, true, 8192>(tbase + TM_U, sb + OFF_T, sb + OFF_V, ID_KxMN, false);
                    mma_commit(&bar_u);
                }
            }
            ok = named_bar_and(kBarSerial, kSerialThreads, ok);
            if (!ok) break;
            {
                // S <- Diag(e^{Gam_63}) S in TMEM (gamma was published before T/P/Kb)
                float sv[64];
                tmem_ld64(tlane + TM_S + 64 * colhalf, sv);
                const float gc = s_gamma[par][32 * quarter + lane];
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    const float2 d = mul2(make_float2(sv[j], sv[j + 1]), make_float2(gc, gc));
                    sv[j] = d.x;
                    sv[j + 1] = d.y;
                }
#pragma unroll
                for (int cb = 0; cb < 64; cb += 16) tmem_st16(tlane + TM_S + 64 * colhalf + cb, sv + cb);
                tmem_wait_st();
            }
            ok = mbar_wait(&bar_u, par, p.timeout_ns);
            tc_fence_after_sync();
            ok = named_bar_and(kBarSerial, kSerialThreads, ok);
            if (!ok) break;
            // U (lanes 0-31 tokens 0-31, lanes 64-95 tokens 32-63) -> bf16, in place over Y
            if ((quarter & 1) == 0) {
                const int tj = 32 * (quarter >> 1) + lane;
                float u[64];
                tmem_ld64(tlane + TM_U + 64 * colhalf, u);
#pragma unroll
                for (int j = 0; j < 64; j += 8)
                    *reinterpret_cast<uint4*>(sm + OFF_V + sw128_offset(tj, 64 * colhalf + j, 8192)) = pack8(u + j);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar_sync(kBarSerial, kSerialThreads);
            // ---- S3: O = Qt S + P U (onto the Qt lanes of TM_C); S <- decayed S + Kb^T U
            if (stid == 0) {
                tc_fence_after_sync();
                issue_mma<4, false, 0, true, 8192>(tbase + TM_C, sb + OFF_P, sb + OFF_V, ID_KxMN, true);
                issue_mma<4, true, 8192, true, 8192>(tbase + TM_S, sb + OFF_KBAR, sb + OFF_V, ID_MNxMN, true);
                mma_commit(&bar_os);
            }
            ok = mbar_wait(&bar_os, par, p.timeout_ns);
            tc_fence_after_sync();
            ok = named_bar_and(kBarSerial, kSerialThreads, ok);
            if (!ok) break;
            // ---- S4: S -> bf16 tile (the next chunk's MMA3 waits on it); O read out of TMEM before
            // MMA3 may overwrite it and staged in the v tile (free now), which a TMA store writes out
            {
                const int i = 32 * quarter + lane;
                float sv[64];
                tmem_ld64(tlane + TM_S + 64 * colhalf, sv);
#pragma unroll
                for (int j = 0; j < 64; j += 8)
                    *reinterpret_cast<uint4*>(sm + OFF_SB + sw128_offset(i, 64 * colhalf + j, 16384)) = pack8(sv + j);
                // the state after a multiple of the interval (only a full chunk can end on one)
                if (p.n_mid > 0 && t0 + kC <= T && (t0 + kC) % p.interval == 0 && i < p.dk && 64 * colhalf < p.dv) {
                    float* dst = p.S_mid + (((size_t)bh * p.n_mid + (t0 + kC) / p.interval - 1) * p.dk + i) * p.dv + 64 * colhalf;
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        __stcs(reinterpret_cast<float4*>(dst + j), make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]));
                }
            }
            // A packed sequence's partial last chunk is written row by row: the rows past its end
            // belong to the next sequence, which a tile store would overwrite
            const bool row_stores = kPacked && t0 + kC > T;
            if ((quarter & 1) == 0) {
                const int r = 32 * (quarter >> 1) + lane;   // token row of the chunk
                float ov[64];
                tmem_ld64(tlane + TM_C + 64 * colhalf, ov);   // warp-collective
                if (kFused) {   // O of the raw q row: O' = O / |q|
                    const float nq = s_norm[par][r];
#pragma unroll
                    for (int j = 0; j < 64; j += 2) {
                        const float2 x = mul2(make_float2(ov[j], ov[j + 1]), make_float2(nq, nq));
                        ov[j] = x.x;
                        ov[j + 1] = x.y;
                    }
                }
                if (row_stores) {
                    if (t0 + r < T && 64 * colhalf < p.dv) {
                        uint4* orow = reinterpret_cast<uint4*>(p.o + ((row0 + t0 + r) * p.H + h) * p.dv + 64 * colhalf);
#pragma unroll
                        for (int j = 0; j < 8; ++j) orow[j] = pack8(ov + 8 * j);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; j += 8)
                        *reinterpret_cast<uint4*>(sm + OFF_V + sw128_offset(r, 64 * colhalf + j, 8192)) = pack8(ov + j);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar_sync(kBarSerial, kSerialThreads);
            if (stid == 32) {
                // rows past the tensor's T are clipped by the tensor map
                if (!row_stores) {
                    tma_store_4d(&tm_o, sm + OFF_V, 0, h, tok0 + t0, bmap);
                    if (p.dv > 64) tma_store_4d(&tm_o, sm + OFF_V + 8192, 64, h, tok0 + t0, bmap);
                    bulk_commit_group();
                }
                if (chunk + 1 < nchunks) {
                    bulk_wait_read_all();   // the staged O is read: the next v may land on it
                    load_v(chunk + 1);
                    pending = chunk + 1;
                }
            }
            if (stid == 0 && chunk + 1 < nchunks) {
                ok = mbar_wait(&bar_kq, par ^ 1u, p.timeout_ns);
                if (ok) issue_for_chunk(chunk + 1);
            }
            if (gate_warp && chunk + 2 < nchunks && !convert_gate(chunk + 2)) ok = false;
        }
        if (!ok && stid == 0) report_status(p.status, KDA_ERR_TIMEOUT);
        if (stid == 32) {
            bulk_wait_all();
            if (pending >= 0) (void)mbar_wait(&bar_v, (uint32_t)(pending & 1), p.timeout_ns);
        }
        if (pending_g >= 0) (void)mbar_wait(&bar_g, (uint32_t)(pending_g & 1), p.timeout_ns);
        if (stid == 0) {
            mma_commit(&bar_drain_s);
            if (!mbar_wait(&bar_drain_s, 0, p.timeout_ns)) report_status(p.status, KDA_ERR_TIMEOUT);
            if (pending_qk >= 0) (void)mbar_wait(&bar_qk, (uint32_t)(pending_qk & 1), p.timeout_ns);
        }
        named_bar_sync(kBarSerial, kSerialThreads);
        tc_fence_after_sync();
        if (ok && p.ST) {
            const int i = 32 * quarter + lane;
            float sv[64];
            tmem_ld64(tlane + TM_S + 64 * colhalf, sv);   // warp-collective
            if (i < p.dk && 64 * colhalf < p.dv) {
                float* dst = p.ST + ((size_t)bh * p.dk + i) * p.dv + 64 * colhalf;
#pragma unroll
                for (int j = 0; j < 64; j += 4)
                    *reinterpret_cast<float4*>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

// [B, T, H, d] bf16 (d = 64 or 128) viewed as a 4-D tensor (d, H, T, B); box = 64 channels x 1 head
// x 64 tokens.  Rows past T read as zeros, which makes the tail of the last chunk an exact no-op, and
// so do channels past d (the box at channel 64 of a 64-wide tensor).
bool make_map(CUtensorMap* m, const void* ptr, int B, int T, int H, int d) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

void* tensor_map_encoder() {
    static void* fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = f;
    });
    return fn;
}

bool prefill_tc_supports(const PrefillArgs& a) {
    return a.dtype == KDA_DTYPE_BF16 && (a.dk == 64 || a.dk == kD) && (a.dv == 64 || a.dv == kD);
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    static std::mutex mu;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 64 && !attr_set[dev]) {
            for (const void* fn : {(const void*)kda_prefill_tc_kernel<false, false>, (const void*)kda_prefill_tc_kernel<true, false>,
                                   (const void*)kda_prefill_tc_kernel<false, true>, (const void*)kda_prefill_tc_kernel<true, true>}) {
                e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
                if (e != cudaSuccess) return e;
            }
            attr_set[dev] = true;
        }
    }
    CUtensorMap mq, mk, mg, mv, mo;
    // packed sequences: one batch entry holding all T tokens
    const int mb = a.cu_seqlens ? 1 : a.B;
    if (!make_map(&mq, a.q, mb, a.T, a.H, a.dk) || !make_map(&mk, a.k, mb, a.T, a.H, a.dk) ||
        !make_map(&mg, a.g, mb, a.T, a.H, a.dk) || !make_map(&mv, a.v, mb, a.T, a.H, a.dv) ||
        !make_map(&mo, a.o, mb, a.T, a.H, a.dv))
        return cudaErrorInvalidValue;
    TcParams prm{static_cast<const __nv_bfloat16*>(a.beta), a.S0, static_cast<__nv_bfloat16*>(a.o), a.ST,
                 a.status, a.timeout_ns, a.skip_handoff, a.S_mid, a.interval, a.n_mid, a.cu_seqlens,
                 a.B, a.T, a.H, a.dk, a.dv};
    const unsigned grid = (unsigned)((size_t)a.B * a.H);
    if (a.cu_seqlens) {
        if (a.fused) kda_prefill_tc_kernel<true, true><<<grid, kThreads, SMEM_DYN, s>>>(mq, mk, mg, mv, mo, prm);
        else kda_prefill_tc_kernel<false, true><<<grid, kThreads, SMEM_DYN, s>>>(mq, mk, mg, mv, mo, prm);
    } else {
        if (a.fused) kda_prefill_tc_kernel<true, false><<<grid, kThreads, SMEM_DYN, s>>>(mq, mk, mg, mv, mo, prm);
        else kda_prefill_tc_kernel<false, false><<<grid, kThreads, SMEM_DYN, s>>>(mq, mk, mg, mv, mo, prm);
    }
    return cudaGetLastError();
}

}  // namespace kda
