// chunk_common.cuh -- pieces shared by the tcgen05 chunk kernels (the
// prefill in chunked_tc.cu and the backward in bwd_tc.cu): bf16 pair
// arithmetic, the compute warps' named barriers, and the UT solve of a
// 64 x 64 unit lower triangular system.  Each including file gets its own
// copy (anonymous namespace).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_common.cuh"

namespace gdr {
namespace {

constexpr int NSP = 68;  // row stride (floats) of the solve's float tiles (16-byte rows)

// Two packed bf16 products, each rounded once to bf16
__device__ __forceinline__ uint32_t mul2(uint32_t x, uint32_t y) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&x),
                               *reinterpret_cast<__nv_bfloat162*>(&y));
    return *reinterpret_cast<uint32_t*>(&r);
}
// Square root to about 1 ulp (one SFU op); its results are rounded to bf16.
__device__ __forceinline__ float sqrt_approx(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Square roots of two packed bf16 (non-negative by contract; a negative
// input gives 0), each rounded to bf16.
__device__ __forceinline__ uint32_t sqrt2(uint32_t x) {
    return tc::pack_bf16x2(sqrt_approx(fmaxf(__uint_as_float(x << 16), 0.f)),
                           sqrt_approx(fmaxf(__uint_as_float(x & 0xFFFF0000u), 0.f)));
}
// Reciprocal to about 1 ulp (one SFU op); its results are rounded to bf16.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// Named barriers: id 1 = the 16 compute warps, id 2 = warps 0-7, id 3 =
// warps 8-15.  (Id 0, __syncthreads, includes the issuing warp.)
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }
// The compute barrier returning the OR of `x` over the 512 compute threads:
// all of them get the same answer, so they leave the chunk loop together even
// when the issuing warp raises the abort flag while they pass the barrier.
__device__ __forceinline__ bool compute_sync_or(bool x) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 512, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)x)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void half_sync(int id) {
    asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}

// ---------------------------------------------------------------- UT solve
// T = (I + N)^{-1}, N = A_kb strictly lower 64 x 64 (float, row stride NSP, in
// NS), by the 2 x 2 block recursion of a unit lower triangular inverse,
//   [[T1, 0], [T21, T2]] with T21 = -T2 N21 T1,
// applied at 16 and at 32 rows: the four 16 x 16 diagonal inverses by
// substitution, then two rounds for the 16 x 16 blocks (1,0) and (3,2), then
// two for the 32 x 32 block below the diagonal.  Run by 256 threads (tid
// 0-255 as passed; barrier id 2).  Each finished block also goes, in bf16,
// into a 64-row operand panel Z3 (128-byte swizzled rows): T - I + DIAG * I,
// i.e. T - I for DIAG = 0 and T + I for DIAG = 2; the blocks above the
// diagonal are not written (the caller keeps them zero).

// One element into the 128-byte swizzled Z3 rows.
__device__ __forceinline__ void z3_put(uint8_t* z3, int row, int col, float v) {
    *reinterpret_cast<__nv_bfloat16*>(z3 + row * 128 + (((col >> 3) ^ (row & 7)) << 4) +
                                      2 * (col & 7)) = __float2bfloat16_rn(v);
}
__device__ __forceinline__ void z3_put2(uint8_t* z3, int row, int col, float v0, float v1) {
    *reinterpret_cast<uint32_t*>(z3 + row * 128 + (((col >> 3) ^ (row & 7)) << 4) +
                                 2 * (col & 7)) = tc::pack_bf16x2(v0, v1);
}

template <int DIAG>
__device__ __forceinline__ void ut_diag(const float* NS, float* TS, uint8_t* z3, int tid) {
    if (tid < 64) {
        // column c of the inverse of diagonal block I: x_r = [r == c] - sum_{s<r} N_rs x_s,
        // each row of N read as 16-byte vectors, two partial sums per row
        const int I = tid >> 4, c = tid & 15;
        const float* nb = NS + (16 * I) * NSP + 16 * I;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            const float* row = nb + r * NSP;
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int s4 = 0; 4 * s4 < r; ++s4) {
                const float4 v = *reinterpret_cast<const float4*>(row + 4 * s4);
                if (4 * s4 + 0 < r) acc0 = fmaf(v.x, x[4 * s4 + 0], acc0);
                if (4 * s4 + 1 < r) acc1 = fmaf(v.y, x[4 * s4 + 1], acc1);
                if (4 * s4 + 2 < r) acc0 = fmaf(v.z, x[4 * s4 + 2], acc0);
                if (4 * s4 + 3 < r) acc1 = fmaf(v.w, x[4 * s4 + 3], acc1);
            }
            x[r] -= acc0 + acc1;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            TS[(16 * I + r) * NSP + 16 * I + c] = x[r];
            z3_put(z3, 16 * I + r, 16 * I + c, r > c ? x[r] : (r == c ? (float)DIAG : 0.f));
        }
    }
    half_sync(2);
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

// d = A(16 x 8KS) B(8KS x 8) for float tiles in shared memory (A at its
// (0,0) with row stride lda, B likewise with ldb).  The block products of
// the solve are tiny and latency-bound, so they use the warp-level mma.sync
// path in tf32 (T is rounded to bf16 afterwards); the chunk's large products
// stay on tcgen05.  Fragments: g = lane/4, t = lane%4; A rows g, g+8 and
// columns t, t+4; B rows t, t+4 and column g; D rows g, g+8, columns 2t, 2t+1.
template <int KS>
__device__ __forceinline__ void tile_16x8(float* d, const float* A, int lda, const float* Bm,
                                          int ldb, int g, int t) {
    d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const float* a0 = A + g * lda + 8 * ks + t;
        const float* b0 = Bm + (8 * ks + t) * ldb + g;
        const uint32_t af[4] = {to_tf32(a0[0]), to_tf32(a0[8 * lda]), to_tf32(a0[4]),
                                to_tf32(a0[8 * lda + 4])};
        const uint32_t bfr[2] = {to_tf32(b0[0]), to_tf32(b0[4 * ldb])};
        mma_tf32_16x8x8(d, af, bfr);
    }
}

template <int DIAG>
__device__ __forceinline__ void ut_solve(float* NS, float* TS, float* PS, uint8_t* z3, int tid) {
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    ut_diag<DIAG>(NS, TS, z3, tid);
    // blocks (1,0) and (3,2): P = N_IJ T_JJ, then T_IJ = -T_II P (warps 0-3)
    const int b = warp >> 1, nt = warp & 1;
    const int I = 2 * b + 1, J = 2 * b;
    float d[4];
    if (warp < 4) {
        tile_16x8<2>(d, NS + (16 * I) * NSP + 16 * J, NSP, TS + (16 * J) * NSP + 16 * J + 8 * nt,
                     NSP, g, t);
        float* pp = PS + b * 256 + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(pp + g * 16) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(pp + (g + 8) * 16) = make_float2(d[2], d[3]);
    }
    half_sync(2);
    if (warp < 4) {
        tile_16x8<2>(d, TS + (16 * I) * NSP + 16 * I, NSP, PS + b * 256 + 8 * nt, 16, g, t);
        const int row = 16 * I + g, col = 16 * J + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(TS + row * NSP + col) = make_float2(-d[0], -d[1]);
        *reinterpret_cast<float2*>(TS + (row + 8) * NSP + col) = make_float2(-d[2], -d[3]);
        z3_put2(z3, row, col, -d[0], -d[1]);
        z3_put2(z3, row + 8, col, -d[2], -d[3]);
    }
    half_sync(2);
    // Y = N21 T1 (rows 32-63 of N, columns 0-31), kept in the unused upper
    // right quadrant of NS: block (i, j) sums over the blocks s = j..1 of T1.
    const int i2 = warp >> 2, j2 = (warp >> 1) & 1;
    {
        const float* A = NS + (32 + 16 * i2) * NSP + 16 * j2;
        const float* Bm = TS + (16 * j2) * NSP + 16 * j2 + 8 * nt;
        if (j2 == 0) tile_16x8<4>(d, A, NSP, Bm, NSP, g, t);
        else tile_16x8<2>(d, A, NSP, Bm, NSP, g, t);
        float* yp = NS + (16 * i2 + g) * NSP + 32 + 16 * j2 + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(yp) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(yp + 8 * NSP) = make_float2(d[2], d[3]);
    }
    half_sync(2);
    // T21 = -T2 Y: block (i, j) sums T2[i][s] Y[s][j] over s = 0..i
    {
        const float* A = TS + (32 + 16 * i2) * NSP + 32;
        const float* Bm = NS + 32 + 16 * j2 + 8 * nt;
        if (i2 == 0) tile_16x8<2>(d, A, NSP, Bm, NSP, g, t);
        else tile_16x8<4>(d, A, NSP, Bm, NSP, g, t);
        const int row = 32 + 16 * i2 + g, col = 16 * j2 + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(TS + row * NSP + col) = make_float2(-d[0], -d[1]);
        *reinterpret_cast<float2*>(TS + (row + 8) * NSP + col) = make_float2(-d[2], -d[3]);
        z3_put2(z3, row, col, -d[0], -d[1]);
        z3_put2(z3, row + 8, col, -d[2], -d[3]);
    }
}


}  // namespace
}  // namespace gdr
