// chunked_tc.cu -- chunkwise-parallel gated delta rule on the Blackwell
// tensor cores (tcgen05, accumulators in tensor memory) fed by TMA, bf16
// inputs, float32 state, dk = dv = 128, chunk C = 64.
//
// Chunked form (per chunk of n <= 64 tokens, state S0 at its start,
// gamma_r = prod_{i<=r} a_i per key channel, U = w*V):
//   A_kk[r,s] = sum_c k_rc k_sc gamma_rc/gamma_sc          (strictly lower)
//   A_kb[r,s] = sum_c k_rc b_sc k_sc gamma_rc/gamma_sc     (strictly lower)
//   A_qk[r,s], A_qb[r,s] the same with q_r for k_r          (lower, diagonal in)
//   T  = (I + A_kb)^{-1}                 UT transform (unit lower triangular)
//   R  = Kh S0 + A_kk U,  E = T R        Kh = gamma*K   (row r of E: S'_r^T k_r)
//   O  = Qh S0 + A_qk U - A_qb E,        Qh = gamma*Q
//   S  = gamma_C * S0 + Kt^T U - Bt^T E, Kt = (gamma_C/gamma)*K, Bt = b*Kt
// This is the WY / UT-transform evaluation of the rank-1 Householder-like
// products that the FG^2-GDN page (gist.science 2604.19021) names in section
// 2 "Methodology" (WY chunked training) and section 3 (DPLR structure, KDA
// chunked kernels), derived from the update rule of section 2; decay per
// channel as in KDA (section 1), decoupled erase/write gates as in Gated
// DeltaNet-2 (needhelp.icu, gates table).
//
// Scaling around the middle token m = 31.  With g_m = gamma_m per channel:
//   K' = (gamma/g_m)*K, Q' = (gamma/g_m)*Q, K" = (g_m/gamma)*K, B" = b*K"
// and the state kept as S~ = Diag(g_m) S0, one 128 x 128 accumulator X holds
// [R; O] (rows 0-63 tokens of R, rows 64-127 tokens of O):
//   X   = [K'; Q'] S~ + [A_kk; A_qk] U          (R and the first terms of O)
//   X  += [T - I; 0] R                           (rows 0-63 become E = T R)
//   X  += [0; -A_qb] E                           (rows 64-127 become O)
//   S~ += K"^T U - B"^T E,   S_new = Diag(gamma_C/g_m) S~
// and the grams are [K';Q'] [K";B"]^T.  Every factor is a ratio of decay
// products over at most half a chunk; if one leaves float range (decay
// stronger than about exp(-80) over half a chunk, or an exact zero) the
// kernel sets GDR_ERR_RANGE in the device error word (the float32 CUDA-core
// kernel, chunk <= 32, has no such limit).
//
// One CTA (16 warps) owns one (batch, head) and walks its chunks in order;
// S~ stays in float32 in tensor memory (lane = key channel) for the whole
// sequence.  Raw q/k/v and vector gates arrive by TMA as 64-token x
// 64-channel boxes, 128-byte swizzled, i.e. already in the operand layout of
// tc_common.cuh, each prefetched as soon as its destination is free; o leaves
// by a TMA store.  Products are tcgen05.mma issued by one thread; the decay
// products, the UT solve and the conversions run on the CUDA cores with
// 16-byte shared-memory accesses.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "tc_common.cuh"

namespace gdr {
namespace {

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // dk = dv
constexpr int NT = 512;      // threads per CTA (16 warps)

// ---- shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_RAW = 0;         // raw k (rows 0-63) and q (rows 64-127), 2 panels
constexpr uint32_t OFF_X1 = 32768;      // [K'; Q'] 128 x 128 (raw a, b land here)
constexpr uint32_t OFF_X2 = 65536;      // [K"; B"] 128 x 128
constexpr uint32_t OFF_U = 98304;       // U = w*v [s][j] 64 x 128 (raw v lands here)
constexpr uint32_t OFF_LQ = 114688;     // [A_kk; A_qk] 128 x 64; then R bf16 [s][j] 64 x 128
                                        // (raw w lands here)
constexpr uint32_t OFF_Z3 = 131072;     // [T - I; 0; -A_qb] 192 x 64
constexpr uint32_t OFF_S0 = 155648;     // S~ [i][j] bf16 128 x 128; before it, the next
                                        // chunk's decay factors:
constexpr uint32_t OFF_E1 = OFF_S0;             //  gamma_r/g_m, bf16 [64][128]
constexpr uint32_t OFF_E1I = OFF_S0 + 16384;    //  g_m/gamma_r, bf16 [64][128]
constexpr uint32_t OFF_R = 188416;      // scratch region:
constexpr uint32_t OFF_NS = OFF_R;              //  P4-P5: A_kb, float [64][68]
constexpr uint32_t OFF_TS = OFF_R + 17408;      //  P5: T, float [64][68]
constexpr uint32_t OFF_PS = OFF_R + 34816;      //  P5: float [3][16][16]
constexpr uint32_t OFF_OST = OFF_R;             //  P8: o staging [r][j] 64 x 128
constexpr uint32_t OFF_EB = OFF_R + 16384;      //  P7: E bf16 [s][j] 64 x 128
constexpr uint32_t OFF_SMALL = OFF_R + 37888;   // 226304
constexpr uint32_t OFF_FCUR = OFF_SMALL;        // float[128]: state scale this chunk
constexpr uint32_t OFF_FPREV = OFF_SMALL + 512; // float[128]: gamma_C/g_m of last chunk
constexpr uint32_t OFF_SCA = OFF_SMALL + 1024;  // float[2][3][64]: scalar a, b, w (2 chunks)
constexpr uint32_t OFF_QT = OFF_SMALL + 2560;   // float[4][128]: 16-token group products
constexpr uint32_t OFF_BAR = OFF_SMALL + 4608;  // 4 mbarriers: mma, kq, ab, vw
constexpr uint32_t OFF_TSLOT = OFF_BAR + 32;
constexpr uint32_t OFF_ABORT = OFF_BAR + 36;
constexpr uint32_t SMEM_USED = OFF_BAR + 40;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(OFF_PS + 3 * 256 * 4 <= OFF_SMALL, "solve scratch");

constexpr int NSP = 68;  // row stride (floats) of the solve's float tiles (16-byte rows)

// ---- tensor-memory columns (512 allocated)
constexpr uint32_t TM_G = 0;     // gram 128 x 128
constexpr uint32_t TM_X = 128;   // [R -> E; O] 128 x 128
constexpr uint32_t TM_S = 256;   // S~ 128 x 128 (lane = key channel), float32 state

constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr uint32_t BOX_BYTES = 64 * 128;     // one 64 x 64 bf16 TMA box
constexpr uint32_t IDESC_NEG_B = 1u << 14;   // negate the B operand

struct TcMaps {
    CUtensorMap q, k, v, a, b, w, o;  // a/b/w only meaningful for vector gates
};

// 8 floats -> 8 bf16 (one 16-byte chunk)
__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    u.x = tc::pack_bf16x2(f[0], f[1]);
    u.y = tc::pack_bf16x2(f[2], f[3]);
    u.z = tc::pack_bf16x2(f[4], f[5]);
    u.w = tc::pack_bf16x2(f[6], f[7]);
    return u;
}
// 8 packed bf16 products, each rounded once to bf16
__device__ __forceinline__ uint32_t mul2(uint32_t x, uint32_t y) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&x),
                               *reinterpret_cast<__nv_bfloat162*>(&y));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint4 mul8(uint4 x, uint4 y) {
    return make_uint4(mul2(x.x, y.x), mul2(x.y, y.y), mul2(x.z, y.z), mul2(x.w, y.w));
}
__device__ __forceinline__ uint4 splat8(float v) {
    const uint32_t p = tc::pack_bf16x2(v, v);
    return make_uint4(p, p, p, p);
}
// Reciprocal to about 1 ulp (one SFU op); its results are rounded to bf16.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// Barrier over one half of the CTA: id 1 = warps 0-7, id 2 = warps 8-15.
__device__ __forceinline__ void half_sync(int id) {
    asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}

// ---------------------------------------------------------------- UT solve
// T = (I + N)^{-1}, N strictly lower 64 x 64 in NS, T into TS (both float,
// row stride NSP); run by warps 0-7 (barrier id 1).  The four 16 x 16 diagonal blocks by right-looking
// substitution, then the off-diagonal blocks level by level:
//   T_IJ = -T_II * P,  P = sum_{s in blocks J..I-1} N[I rows][s] T[s][J cols].
__device__ __forceinline__ void ut_diag(const float* NS, float* TS, int tid) {
    if (tid < 64) {
        const int I = tid >> 4, c = tid & 15;
        const float* nb = NS + (16 * I) * NSP + 16 * I;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
            const float xs = x[s];
#pragma unroll
            for (int r = s + 1; r < 16; ++r) x[r] = fmaf(-nb[r * NSP + s], xs, x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) TS[(16 * I + r) * NSP + 16 * I + c] = x[r];
    }
    half_sync(1);
}

// tf32 operand of mma.sync (round to nearest, ties away)
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D(16x8) += A(16x8) B(8x8), tf32 inputs, float32 accumulate (one warp).
__device__ __forceinline__ void mma_tf32_16x8x8(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One level: blocks (I, J = I - LVL), each 16 x 16, two warps per block (one
// per 8-column half).  The 16 x 16 x 16k block products are tiny and
// latency-bound, so they use the warp-level mma.sync tensor path in tf32
// (T is rounded to bf16 afterwards); the chunk's large products stay on
// tcgen05.  Fragments: g = lane/4, t = lane%4; A rows g, g+8 and columns
// t, t+4; B rows t, t+4 and column g; D rows g, g+8 and columns 2t, 2t+1.
template <int LVL>
__device__ __forceinline__ void ut_level(const float* NS, float* TS, float* PS, int tid) {
    constexpr int NB = 4 - LVL;
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int b = warp >> 1, nt = warp & 1;
    const bool on = warp < 2 * NB;
    const int I = LVL + b, J = b;
    if (on) {
        // P[:, 8nt..8nt+7] = N[I rows][16J .. 16I) T[16J .. 16I)[J cols]
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        const float* n0 = NS + (16 * I + g) * NSP + 16 * J + t;
        const float* t0 = TS + (16 * J + t) * NSP + 16 * J + 8 * nt + g;
#pragma unroll
        for (int ks = 0; ks < 2 * LVL; ++ks) {
            const uint32_t af[4] = {to_tf32(n0[8 * ks]), to_tf32(n0[8 * NSP + 8 * ks]),
                                    to_tf32(n0[8 * ks + 4]), to_tf32(n0[8 * NSP + 8 * ks + 4])};
            const uint32_t bfr[2] = {to_tf32(t0[(8 * ks) * NSP]), to_tf32(t0[(8 * ks + 4) * NSP])};
            mma_tf32_16x8x8(d, af, bfr);
        }
        float* pp = PS + b * 256 + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(pp + g * 16) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(pp + (g + 8) * 16) = make_float2(d[2], d[3]);
    }
    half_sync(1);
    if (on) {
        // T_IJ[:, 8nt..] = -T_II P[:, 8nt..]
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        const float* a0p = TS + (16 * I + g) * NSP + 16 * I + t;
        const float* b0p = PS + b * 256 + t * 16 + 8 * nt + g;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const uint32_t af[4] = {to_tf32(a0p[8 * ks]), to_tf32(a0p[8 * NSP + 8 * ks]),
                                    to_tf32(a0p[8 * ks + 4]), to_tf32(a0p[8 * NSP + 8 * ks + 4])};
            const uint32_t bfr[2] = {to_tf32(b0p[(8 * ks) * 16]), to_tf32(b0p[(8 * ks + 4) * 16])};
            mma_tf32_16x8x8(d, af, bfr);
        }
        float* tp = TS + (16 * I + g) * NSP + 16 * J + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(tp) = make_float2(-d[0], -d[1]);
        *reinterpret_cast<float2*>(tp + 8 * NSP) = make_float2(-d[2], -d[3]);
    }
    half_sync(1);
}

// ---------------------------------------------------------------- TMA issue
// Group "kq": raw k and q into RAW.  Group "ab": vector a and b into X1.
// Group "vw": v into U and vector w into LQ.
__device__ __forceinline__ void issue_kq(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                         uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 4 * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384, &m.k, 64 * p, hi, t0, bi, bar);
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384 + 8192, &m.q, 64 * p, hi, t0, bi, bar);
    }
}

__device__ __forceinline__ void issue_ab(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                         bool va, bool vb, uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 2u * ((va ? 1u : 0u) + (vb ? 1u : 0u)) * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        if (va) tc::tma_load_4d(sbase + OFF_X1 + p * 16384, &m.a, 64 * p, hi, t0, bi, bar);
        if (vb) tc::tma_load_4d(sbase + OFF_X1 + p * 16384 + 8192, &m.b, 64 * p, hi, t0, bi, bar);
    }
}

__device__ __forceinline__ void issue_vw(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                         bool vw, uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 2u * (1u + (vw ? 1u : 0u)) * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        tc::tma_load_4d(sbase + OFF_U + p * 8192, &m.v, 64 * p, hi, t0, bi, bar);
        if (vw) tc::tma_load_4d(sbase + OFF_LQ + p * 8192, &m.w, 64 * p, hi, t0, bi, bar);
    }
}

// Decay factors of one chunk, run by warps 8-15 (barrier id 2; u = tid - 256):
// per key channel the products gamma_r of a over the chunk, g_m = gamma_31,
// written as bf16 pairs gamma_r/g_m (E1) and g_m/gamma_r (E1I) [64][128];
// fcur = fprev * g_m (scale of S~ this chunk), fprev = gamma_63/g_m; and the
// range check of the factorisation.  Thread (pair p2 of channels, quarter q4)
// walks 16 tokens.
__device__ __forceinline__ void decay_pass(uint8_t* sm, int u, bool va, int a_kind, int n,
                                           const float* sca_a, float* QT, float* fcur,
                                           float* fprev, int* err_word) {
    const int p2 = u & 63, q4 = u >> 6;
    const uint32_t aoff = (uint32_t)(p2 >> 5) * 16384u + 4u * (uint32_t)(p2 & 3);
    const int ach = (p2 & 31) >> 2;
    float loc0[16], loc1[16];
    float run0 = 1.f, run1 = 1.f;
#pragma unroll
    for (int x = 0; x < 16; ++x) {
        const int r = 16 * q4 + x;
        float a0, a1;
        if (va) {
            const uint32_t pr = *reinterpret_cast<const uint32_t*>(
                sm + OFF_X1 + aoff + (uint32_t)r * 128u + ((uint32_t)(ach ^ (r & 7)) << 4));
            a0 = __uint_as_float(pr << 16);
            a1 = __uint_as_float(pr & 0xFFFF0000u);
        } else {
            a0 = a1 = sca_a[r];
        }
        const bool live = a_kind != GDR_GATE_ONE && r < n;
        run0 *= live ? a0 : 1.f;
        run1 *= live ? a1 : 1.f;
        loc0[x] = run0;
        loc1[x] = run1;
    }
    *reinterpret_cast<float2*>(QT + q4 * D + 2 * p2) = make_float2(run0, run1);
    half_sync(2);
    float pre0 = 1.f, pre1 = 1.f, gm0 = 1.f, gm1 = 1.f, gc0 = 1.f, gc1 = 1.f;
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
        const float2 qv = *reinterpret_cast<const float2*>(QT + gg * D + 2 * p2);
        if (gg < q4) { pre0 *= qv.x; pre1 *= qv.y; }
        if (gg < 2) { gm0 *= qv.x; gm1 *= qv.y; } else { gc0 *= qv.x; gc1 *= qv.y; }
    }
    const float f0 = pre0 * rcp_approx(gm0), f1 = pre1 * rcp_approx(gm1);
#pragma unroll
    for (int x = 0; x < 16; ++x) {
        const int r = 16 * q4 + x;
        const float e0 = loc0[x] * f0, e1v = loc1[x] * f1;
        *reinterpret_cast<uint32_t*>(sm + OFF_E1 + r * 256 + 4 * p2) = tc::pack_bf16x2(e0, e1v);
        *reinterpret_cast<uint32_t*>(sm + OFF_E1I + r * 256 + 4 * p2) =
            tc::pack_bf16x2(rcp_approx(e0), rcp_approx(e1v));
    }
    if (q4 == 0) {
        const int i = 2 * p2;
        fcur[i] = fprev[i] * gm0;
        fcur[i + 1] = fprev[i + 1] * gm1;
        fprev[i] = gc0;
        fprev[i + 1] = gc1;
        // the largest factors, gamma_0/g_m and g_m/gamma_63, must stay in range
        const bool ok0 = gm0 > 0.f && loc0[0] <= gm0 * 1e35f && gc0 >= 1e-35f;
        const bool ok1 = gm1 > 0.f && loc1[0] <= gm1 * 1e35f && gc1 >= 1e-35f;
        if (a_kind != GDR_GATE_ONE && !(ok0 && ok1)) atomicOr(err_word, kErrRange);
    }
}

// One thread waits on `bar`; the CTA barrier that follows releases the rest.
__device__ __forceinline__ void wait_then_sync(uint32_t bar, uint32_t parity, int tid,
                                               volatile int* abort_s) {
    if (tid == 0 && !tc::mbar_wait_bounded(bar, parity, WAIT_NS)) *abort_s = 1;
    __syncthreads();
    tc::fence_after_sync();
}

__global__ void __launch_bounds__(NT, 1)
chunked_tc_kernel(const __grid_constant__ TcMaps maps, int B, int T, int H,
                  const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                  const __nv_bfloat16* __restrict__ w, int a_kind, int b_kind, int w_kind,
                  const float* __restrict__ s0, float* __restrict__ s_final,
                  int* __restrict__ err_word) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float* QT = reinterpret_cast<float*>(sm + OFF_QT);
    float* NS = reinterpret_cast<float*>(sm + OFF_NS);
    float* TS = reinterpret_cast<float*>(sm + OFF_TS);
    float* PS = reinterpret_cast<float*>(sm + OFF_PS);
    float* fcur = reinterpret_cast<float*>(sm + OFF_FCUR);
    float* fprev = reinterpret_cast<float*>(sm + OFF_FPREV);
    float* sca_all = reinterpret_cast<float*>(sm + OFF_SCA);  // [2][3][64]
    volatile int* abort_s = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
    const uint32_t bar_mma = sbase + OFF_BAR;
    const uint32_t bar_kq = sbase + OFF_BAR + 8;
    const uint32_t bar_ab = sbase + OFF_BAR + 16;
    const uint32_t bar_vw = sbase + OFF_BAR + 24;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quarter = warp & 3;                  // tensor-memory lanes 32*quarter ..
    const int cb = warp >> 2;                      // 32-column block this warp reads
    const int lane_t = 32 * quarter + (tid & 31);  // tensor-memory lane of this thread
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;

    const int bh = blockIdx.x;
    const int bi = bh / H, hi = bh % H;
    const size_t soff = (size_t)bh * D * D;
    const bool va = a_kind == GDR_GATE_VECTOR, vb = b_kind == GDR_GATE_VECTOR,
               vw = w_kind == GDR_GATE_VECTOR;
    const bool has_ab = va || vb;

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_kq, 1);
        tc::mbar_init(bar_ab, 1);
        tc::mbar_init(bar_vw, 1);
        tc::mbar_fence_init();
        *abort_s = 0;
        tc::tma_prefetch_desc(&maps.q);
        tc::tma_prefetch_desc(&maps.k);
        tc::tma_prefetch_desc(&maps.v);
        tc::tma_prefetch_desc(&maps.o);
    }
    if (tid < D) fprev[tid] = 1.0f;
    // the middle 64 rows of Z3 stay zero for the whole sequence
    *reinterpret_cast<uint4*>(sm + OFF_Z3 + 8192 + 16 * tid) = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 0) tc::tmem_alloc(sbase + OFF_TSLOT, 512);
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TSLOT);
    uint32_t ph_mma = 0, ph_kq = 0, ph_ab = 0, ph_vw = 0;

    if (tid == 0 && T > 0) {
        issue_kq(maps, sbase, 0, hi, bi, bar_kq);
        if (has_ab) issue_ab(maps, sbase, 0, hi, bi, va, vb, bar_ab);
        issue_vw(maps, sbase, 0, hi, bi, vw, bar_vw);
    }
    // scalar gates of chunk starting at t0n into buffer `buf` (1.0 past T)
    auto load_scalars = [&](int t0n, int buf) {
        if (tid < C) {
            const int nn = min(C, T - t0n);
            const long long tok = ((long long)bi * T + t0n + tid) * H + hi;
            const bool in = tid < nn;
            float* sc = sca_all + buf * 192;
            sc[tid] = (a_kind == GDR_GATE_SCALAR && in) ? to_f32(a[tok]) : 1.f;
            sc[64 + tid] = (b_kind == GDR_GATE_SCALAR && in) ? to_f32(b[tok]) : 1.f;
            sc[128 + tid] = (w_kind == GDR_GATE_SCALAR && in) ? to_f32(w[tok]) : 1.f;
        }
    };
    if (T > 0) load_scalars(0, 0);

    // ---- initial state S0 (unscaled) into tensor memory: lane i, columns j
    {
        const int c0 = 32 * cb;
        float vals[32];
        if (s0) {
            const float4* src = reinterpret_cast<const float4*>(s0 + soff + (size_t)lane_t * D + c0);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float4 v4 = src[x];
                vals[4 * x] = v4.x; vals[4 * x + 1] = v4.y; vals[4 * x + 2] = v4.z; vals[4 * x + 3] = v4.w;
            }
        } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) vals[x] = 0.f;
        }
        tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
        tc::tmem_wait_st();
    }
    tc::fence_before_sync();
    __syncthreads();
    // decay factors of the first chunk (later chunks get theirs under the
    // previous chunk's UT solve)
    if (T > 0 && warp >= 8) {
        if (tid == 256 && has_ab && !tc::mbar_wait_bounded(bar_ab, ph_ab, WAIT_NS)) *abort_s = 1;
        half_sync(2);
        decay_pass(sm, tid - 256, va, a_kind, min(C, T), sca_all, QT, fcur, fprev, err_word);
    }
    ph_ab ^= (T > 0 && has_ab) ? 1 : 0;
    __syncthreads();

#pragma unroll 1
    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        const bool has_next = t0 + C < T;
        const int cur = (t0 / C) & 1;
        const float* sca = sca_all + cur * 192;

        // ================= P1: wait for the chunk's tiles, scaled operands
        if (tid == 0) {
            tc::bulk_wait_read();  // the previous o store has left the staging tile
            bool ok = tc::mbar_wait_bounded(bar_kq, ph_kq, WAIT_NS);
            ok = ok && tc::mbar_wait_bounded(bar_vw, ph_vw, WAIT_NS);
            if (!ok) *abort_s = 1;
        }
        ph_kq ^= 1;
        ph_vw ^= 1;
        __syncthreads();
        // ================= P1c:
        {
            // K' = e1*k, Q' = e1*q, K" = k/e1, B" = b*K", U = w*v, 8 channels
            // (16 bytes) per access, packed bf16 products
#pragma unroll 1
            for (int it = tid; it < C * 16; it += NT) {
                const int r = it >> 4, c16 = it & 15, p = c16 >> 3, ch = c16 & 7;
                const uint32_t swz = ((uint32_t)(ch ^ (r & 7)) << 4) + (uint32_t)r * 128u;
                const uint32_t otop = (uint32_t)p * 16384u + swz;  // rows 0-63 of 128-row tiles
                const uint32_t obot = otop + 8192u;                // rows 64-127
                const uint32_t o64 = (uint32_t)p * 8192u + swz;    // 64-row tiles
                const uint4 k4 = *reinterpret_cast<const uint4*>(sm + OFF_RAW + otop);
                const uint4 q4 = *reinterpret_cast<const uint4*>(sm + OFF_RAW + obot);
                const uint4 v4 = *reinterpret_cast<const uint4*>(sm + OFF_U + o64);
                const uint4 b4 = vb ? *reinterpret_cast<const uint4*>(sm + OFF_X1 + obot)
                                    : splat8(sca[64 + r]);
                const uint4 w4 = vw ? *reinterpret_cast<const uint4*>(sm + OFF_LQ + o64)
                                    : splat8(sca[128 + r]);
                const uint4 e4 = *reinterpret_cast<const uint4*>(sm + OFF_E1 + r * 256 + 16 * c16);
                const uint4 ei4 = *reinterpret_cast<const uint4*>(sm + OFF_E1I + r * 256 + 16 * c16);
                const uint4 kk1 = mul8(k4, e4);   // K'
                const uint4 kk2 = mul8(k4, ei4);  // K"
                *reinterpret_cast<uint4*>(sm + OFF_X1 + otop) = kk1;
                *reinterpret_cast<uint4*>(sm + OFF_X1 + obot) = mul8(q4, e4);    // Q'
                *reinterpret_cast<uint4*>(sm + OFF_X2 + otop) = kk2;
                *reinterpret_cast<uint4*>(sm + OFF_X2 + obot) = mul8(b4, kk2);  // B"
                *reinterpret_cast<uint4*>(sm + OFF_U + o64) = mul8(w4, v4);     // U
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        if (*abort_s) break;
        if (tid == 0) {
            // the RAW tile is free: fetch the next chunk's k and q now
            if (has_next) issue_kq(maps, sbase, t0 + C, hi, bi, bar_kq);
            // gram [K';Q'] [K";B"]^T needs no state: start it under the rescale
            tc::fence_after_sync();
            const uint32_t idKK = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_G, tc::desc_kmajor(sbase + OFF_X1, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_X2, 16384, kk), idKK, kk > 0);
        }

        // ================= P2: S~ <- f_i S~ (lane i), bf16 copy to smem
        tc::fence_after_sync();
        {
            const int c0 = 32 * cb;
            const float f = fcur[lane_t];
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
            tc::tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) vals[x] *= f;
            tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
            tc::store_row32_bf16(sm + OFF_S0 + (cb >> 1) * 16384, lane_t, cb & 1, vals);
            tc::tmem_wait_st();
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // ================= P3: X = [K';Q'] S~, S~ += K"^T U (gram already issued)
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t idMM = tc::idesc_bf16(128, 128, 1, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_X1, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_S0, 16384, kk), idKM, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_X2, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_U, 8192, kk), idMM, true);
            tc::mma_commit(bar_mma);
        }
        wait_then_sync(bar_mma, ph_mma, tid, abort_s);
        ph_mma ^= 1;
        // X1 is free: fetch the next chunk's vector a and b; its scalar gates
        if (tid == 0 && has_next && has_ab) issue_ab(maps, sbase, t0 + C, hi, bi, va, vb, bar_ab);
        if (has_next) load_scalars(t0 + C, cur ^ 1);

        // ================= P4: read the gram; masked blocks out
        {
            // This warp's 32 x 32 block lies below (mode < 0), on (0) or above
            // (> 0) the diagonal of its 64 x 64 gram block: warp-uniform.
            const int mode = (cb & 1) - (quarter & 1);
            const bool top = lane_t < 64;  // rows of K' (else Q')
            const int r = top ? lane_t : lane_t - 64;
            const int s0c = 32 * (cb & 1);  // first s of this column block
            float vals[32];
            if (mode > 0) {
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] = 0.f;
            } else {
                tc::tmem_ld32(tmem + lane_off + TM_G + 32 * cb, vals);
                tc::tmem_wait_ld();
                if (mode == 0) {
                    // strictly lower for the K' rows, diagonal included for Q'
                    const int lim = top ? r - s0c : r - s0c + 1;
#pragma unroll
                    for (int x = 0; x < 32; ++x) vals[x] = x < lim ? vals[x] : 0.f;
                }
            }
            if (cb < 2) {
                tc::store_row32_bf16(sm + OFF_LQ, lane_t, cb & 1, vals);   // [A_kk; A_qk]
            } else if (top) {
                float* nrow = NS + r * NSP + s0c;
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    st4(nrow + x, make_float4(vals[x], vals[x + 1], vals[x + 2], vals[x + 3]));
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] = -vals[x];
                tc::store_row32_bf16(sm + OFF_Z3, 128 + r, cb & 1, vals);  // -A_qb
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        // X += [A_kk; A_qk] U: runs under the solve
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_LQ, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_U, 8192, kk), idKM, true);
            tc::mma_commit(bar_mma);
        }
        if (*abort_s) break;

        // ================= P5: warps 0-7: UT transform T = (I + A_kb)^{-1};
        //                       warps 8-15: R -> bf16, next chunk's decay factors
        if (warp < 8) {
            ut_diag(NS, TS, tid);
            ut_level<1>(NS, TS, PS, tid);
            ut_level<2>(NS, TS, PS, tid);
            ut_level<3>(NS, TS, PS, tid);
            {
                const int r = tid >> 2, c4 = tid & 3;  // T - I, 64 rows x 4 x 16 columns
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int ch = 2 * c4 + hh;
                    float vals[8];
                    const float* trow = TS + r * NSP + 8 * ch;
#pragma unroll
                    for (int x = 0; x < 8; ++x) vals[x] = (8 * ch + x < r) ? trow[x] : 0.f;
                    *reinterpret_cast<uint4*>(sm + OFF_Z3 + r * 128 + ((ch ^ (r & 7)) << 4)) = pack8(vals);
                }
            }
            tc::fence_async_smem();
        } else {
            if (tid == 256 && !tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS)) *abort_s = 1;
            half_sync(2);
            tc::fence_after_sync();
            if (quarter < 2) {   // lanes 0-63 of X hold R; each warp takes 64 columns
                const int c0 = 64 * (cb - 2);
                float vals[32];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    tc::tmem_ld32(tmem + lane_off + TM_X + c0 + 32 * hh, vals);
                    tc::tmem_wait_ld();
                    tc::store_row32_bf16(sm + OFF_LQ + (c0 >> 6) * 8192, lane_t, hh, vals);
                }
            }
            tc::fence_async_smem();
            if (has_next) {
                if (tid == 256 && has_ab &&
                    !tc::mbar_wait_bounded(bar_ab, ph_ab, WAIT_NS)) *abort_s = 1;
                half_sync(2);
                decay_pass(sm, tid - 256, va, a_kind, min(C, T - t0 - C), sca_all + (cur ^ 1) * 192,
                           QT, fcur, fprev, err_word);
            }
        }
        ph_mma ^= 1;
        ph_ab ^= (has_next && has_ab) ? 1 : 0;
        tc::fence_before_sync();
        __syncthreads();

        // ================= P6: X += [T - I; 0] R (rows 0-63 become E)
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_Z3, 8192, kk),
                             tc::desc_mnmajor(sbase + OFF_LQ, 8192, kk), idKM, true);
            tc::mma_commit(bar_mma);
        }
        wait_then_sync(bar_mma, ph_mma, tid, abort_s);
        ph_mma ^= 1;
        // U and LQ are free: fetch the next chunk's v and vector w
        if (tid == 0 && has_next) issue_vw(maps, sbase, t0 + C, hi, bi, vw, bar_vw);

        // ================= P7: E -> bf16; X += [0; -A_qb] E; S~ -= B"^T E
        if (quarter < 2) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_X + 32 * cb, vals);
            tc::tmem_wait_ld();
            tc::store_row32_bf16(sm + OFF_EB + (cb >> 1) * 8192, lane_t, cb & 1, vals);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t idMMn = tc::idesc_bf16(128, 128, 1, 1) | IDESC_NEG_B;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_Z3 + 8192, 8192, kk),
                             tc::desc_mnmajor(sbase + OFF_EB, 8192, kk), idKM, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_X2 + 8192, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_EB, 8192, kk), idMMn, true);
            tc::mma_commit(bar_mma);
        }
        wait_then_sync(bar_mma, ph_mma, tid, abort_s);
        ph_mma ^= 1;

        // ================= P8: O (rows 64-127 of X) -> staging tile -> TMA store
        if (quarter >= 2) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_X + 32 * cb, vals);
            tc::tmem_wait_ld();
            tc::store_row32_bf16(sm + OFF_OST + (cb >> 1) * 8192, lane_t - 64, cb & 1, vals);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_4d(&maps.o, sbase + OFF_OST, 0, hi, t0, bi);
            tc::tma_store_4d(&maps.o, sbase + OFF_OST + 8192, 64, hi, t0, bi);
            tc::bulk_commit();
        }
        if (*abort_s) break;
    }

    if (tid == 0) tc::bulk_wait_all();
    if (*abort_s) {
        atomicOr(err_word, kErrTimeout);
        // let products and copies still in flight land before memory is freed
        if (tid == 0) {
            tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS);
            tc::mbar_wait_bounded(bar_kq, ph_kq, WAIT_NS);
            if (has_ab) tc::mbar_wait_bounded(bar_ab, ph_ab, WAIT_NS);
            tc::mbar_wait_bounded(bar_vw, ph_vw, WAIT_NS);
        }
        __syncthreads();
    } else if (s_final) {
        tc::fence_after_sync();
        const int c0 = 32 * cb;
        const float f = fprev[lane_t];
        float vals[32];
        tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
        tc::tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(s_final + soff + (size_t)lane_t * D + c0);
#pragma unroll
        for (int x = 0; x < 8; ++x)
            dst[x] = make_float4(vals[4 * x] * f, vals[4 * x + 1] * f, vals[4 * x + 2] * f,
                                 vals[4 * x + 3] * f);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_free(tmem, 512);
    }
}

// ---- host side: tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [B, T, H, 128] bf16 tensor as a 4-D map {128, H, T, B}, box {64, 1, 64, 1},
// 128-byte swizzle; rows past T read as zero and are not written.
bool make_map(CUtensorMap* m, const void* ptr, int B, int T, int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                                   (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

bool chunked_tc_supports(const gdr_desc& d) {
    return d.in_dtype == GDR_BF16 && d.dk == D && d.dv == D && d.chunk == C;
}

cudaError_t launch_chunked_tc(const gdr_desc& d, const void* q, const void* k, const void* v,
                              const void* a, const void* b, const void* w, const float* s0,
                              void* o, float* s_final, int* err_word, cudaStream_t st) {
    TcMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (d.T > 0) {
        bool ok = make_map(&maps.q, q, d.B, d.T, d.H) && make_map(&maps.k, k, d.B, d.T, d.H) &&
                  make_map(&maps.v, v, d.B, d.T, d.H) && make_map(&maps.o, o, d.B, d.T, d.H);
        if (ok && d.decay == GDR_GATE_VECTOR) ok = make_map(&maps.a, a, d.B, d.T, d.H);
        if (ok && d.erase == GDR_GATE_VECTOR) ok = make_map(&maps.b, b, d.B, d.T, d.H);
        if (ok && d.write == GDR_GATE_VECTOR) ok = make_map(&maps.w, w, d.B, d.T, d.H);
        if (!ok) return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(chunked_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunked_tc_kernel<<<(unsigned)(d.B * d.H), NT, SMEM_BYTES, st>>>(
        maps, d.B, d.T, d.H, (const __nv_bfloat16*)a, (const __nv_bfloat16*)b,
        (const __nv_bfloat16*)w, (int)d.decay, (int)d.erase, (int)d.write, s0, s_final,
        err_word);
    return cudaGetLastError();
}

}  // namespace gdr
