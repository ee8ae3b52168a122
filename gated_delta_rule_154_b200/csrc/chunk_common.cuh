// chunk_common.cuh -- pieces shared by the tcgen05 chunk kernels (the
// prefill in chunked_tc.cu and the backward in bwd_tc.cu): bf16 pair
// arithmetic, the compute warps' named barriers, and the UT solve of a
// 64 x 64 unit lower triangular system.  Each including file gets its own
// copy (anonymous namespace).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
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

// ------------------------------------------------------------ operand pass

// Tile offsets (bytes from the shared-memory base) of one operand pass: the
// raw tiles it reads and the operand tiles it writes.  q, k, a, b and Q', K',
// K", B" are halves of 128-row tiles (16 KB panels); v (replaced by U) and w
// are 64-row tiles (8 KB panels).
struct OpTiles {
    uint32_t q, k, a, b, Qp, Kp, Kpp, Bpp, v, w;
};

// Byte offset of the 8-byte group of channels 4cq .. 4cq+3 in row r of a
// tile with `pb`-byte panels (128-byte swizzled rows).
__device__ __forceinline__ uint32_t quad_off(int r, int cq, uint32_t pb) {
    return (uint32_t)(cq >> 4) * pb + (uint32_t)r * 128u +
           ((uint32_t)(((cq & 15) >> 1) ^ (r & 7)) << 4) + 8u * (uint32_t)(cq & 1);
}
__device__ __forceinline__ uint2 mul4(uint2 x, uint2 y) {
    return make_uint2(mul2(x.x, y.x), mul2(x.y, y.y));
}
__device__ __forceinline__ uint2 sqrt4(uint2 x) { return make_uint2(sqrt2(x.x), sqrt2(x.y)); }
__device__ __forceinline__ uint2 ld8(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ void st8(uint8_t* p, uint2 v) { *reinterpret_cast<uint2*>(p) = v; }
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Decay factors and scaled operands of one 64-token chunk, all 512 compute
// threads.  Thread (token octet q8 = warp / 2, channel quad cq = 16 (warp %
// 2) + lane / 2, half h = lane % 2) reads the decays of its four channels
// over its four tokens of the octet (8-byte accesses; a warp covers two
// 64-channel row halves per access), forms their running products (leaving
// out the chunk's first token, so that no divisor below holds a_0), takes the
// other half's product from the neighbouring lane, and for h = 0 writes the
// octet totals (QT, float [8][128]).  After one exchange it has gamma_r / g_m and
// g_m / gamma_r (g_m = gamma_31) for its four tokens (8 q8 + 4 h ..) and
// writes, one 8-byte group per token and tensor,
//   Q' = (gamma/g_m) q, K' = (gamma/g_m) k, K" = (g_m/gamma) k, B" = b K",
//   U = w v                                       (each rounded once to bf16)
// in place over the raw tiles.  Every divisor is a product of a over tokens
// 1..31 or 32..63 of the chunk (or a part of one); the octet-0 threads of
// warp 0 check that the two whole products stay at or above 1e-35 and hand
// each channel's g_m and gc = gamma_63/g_m to chan(i, g_m, gc).  `mid` runs
// between the two halves (after the exchange barrier), before any operand
// tile is written.  PACKED: rows past n are zeroed (k, q, v) instead of left
// to the TMA fill.  FG2: key sqrt(beta^k) k with erase gate 1, write gate
// sqrt(beta^v).
template <bool PACKED, bool FG2, typename Mid, typename Chan>
__device__ __forceinline__ void operand_pass(uint8_t* sm, const OpTiles tl, int tid, bool va,
                                             bool vb, bool vw, bool fb, bool fw, int a_kind,
                                             int n, const float* sca, float* QT, int* err_word,
                                             Mid&& mid, Chan&& chan) {
    // lane pair (2l, 2l + 1) = the two halves of one (channel quad, octet)
    const int lane = tid & 31, w = tid >> 5;
    const int q8 = w >> 1, h = lane & 1, cq = 16 * (w & 1) + (lane >> 1);
    // this half's decays, four channels per token as packed bf16 (1.0 past
    // the chunk or for GATE_ONE; scalar gates came from bf16, so they are exact)
    uint2 apr[4];
#pragma unroll
    for (int xx = 0; xx < 4; ++xx) {
        const int r = 8 * q8 + 4 * h + xx;
        uint2 pr;
        if (va) {
            pr = ld8(sm + tl.a + quad_off(r, cq, 16384u));
        } else {
            const uint32_t s2 = tc::pack_bf16x2(sca[r], sca[r]);
            pr = make_uint2(s2, s2);
        }
        apr[xx] = (a_kind != GDR_GATE_ONE && r < n) ? pr : make_uint2(0x3F803F80u, 0x3F803F80u);
    }
    // running products over this half (token 0 of the chunk left out), then
    // over the octet with the other half's product
    float own[4] = {1.f, 1.f, 1.f, 1.f};
    float loc[4][4];   // [token of this half][channel]
#pragma unroll
    for (int xx = 0; xx < 4; ++xx) {
        if (8 * q8 + 4 * h + xx > 0) {
            own[0] *= bf_lo(apr[xx].x);
            own[1] *= bf_hi(apr[xx].x);
            own[2] *= bf_lo(apr[xx].y);
            own[3] *= bf_hi(apr[xx].y);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) loc[xx][j] = own[j];
    }
    float run[4], other[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        other[j] = __shfl_xor_sync(0xffffffffu, own[j], 1);
        run[j] = own[j] * other[j];                 // the octet's product
        if (h) {
#pragma unroll
            for (int xx = 0; xx < 4; ++xx) loc[xx][j] *= other[j];
        }
    }
    if (h == 0) {
        const float f0 = q8 == 0 ? bf_lo(apr[0].x) : 1.f, f1 = q8 == 0 ? bf_hi(apr[0].x) : 1.f;
        const float f2 = q8 == 0 ? bf_lo(apr[0].y) : 1.f, f3 = q8 == 0 ? bf_hi(apr[0].y) : 1.f;
        *reinterpret_cast<float4*>(QT + q8 * 128 + 4 * cq) =
            make_float4(f0 * run[0], f1 * run[1], f2 * run[2], f3 * run[3]);
    }
    compute_sync();
    mid();
    // pm: for q8 < 4 the product over the octets after this one up to the
    // middle (sp), for q8 >= 4 over the octets from the middle up to this one
    // (mp)
    float pm[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
    for (int gg = 0; gg < 8; ++gg) {
        if (q8 < 4 ? (gg > q8 && gg < 4) : (gg >= 4 && gg < q8)) {
            const float4 qv = *reinterpret_cast<const float4*>(QT + gg * 128 + 4 * cq);
            pm[0] *= qv.x;
            pm[1] *= qv.y;
            pm[2] *= qv.z;
            pm[3] *= qv.w;
        }
    }
    // this half's tokens from the last: rev = product of a over the octet's
    // tokens after x (for the first half, starting with the second half's)
    float rev[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) rev[j] = h ? 1.f : other[j];
    float dd[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) dd[j] = rcp_approx(pm[j] * run[j]);
#pragma unroll
    for (int xx = 3; xx >= 0; --xx) {
        const int x = 4 * h + xx;          // token of the octet
        const int r = 8 * q8 + x;
        // e = gamma_r/g_m, ei = g_m/gamma_r for the four channels:
        //   r <= 31: e = loc / (run sp), ei = rev sp
        //   r >= 32: e = mp loc,         ei = rev / (mp run)
        float e[4], ei[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (q8 < 4) {
                e[j] = loc[xx][j] * dd[j];
                ei[j] = rev[j] * pm[j];
            } else {
                e[j] = pm[j] * loc[xx][j];
                ei[j] = rev[j] * dd[j];
            }
        }
        const uint2 e4 = make_uint2(tc::pack_bf16x2(e[0], e[1]), tc::pack_bf16x2(e[2], e[3]));
        const uint2 ei4 = make_uint2(tc::pack_bf16x2(ei[0], ei[1]), tc::pack_bf16x2(ei[2], ei[3]));
        const uint32_t o128 = quad_off(r, cq, 16384u), o64 = quad_off(r, cq, 8192u);
        uint2 q4 = ld8(sm + tl.q + o128), k4 = ld8(sm + tl.k + o128), v4 = ld8(sm + tl.v + o64);
        uint2 b4, w4;
        if (vb) {
            b4 = ld8(sm + tl.b + o128);
        } else {
            const uint32_t s2 = tc::pack_bf16x2(sca[64 + r], sca[64 + r]);
            b4 = make_uint2(s2, s2);
        }
        if (vw) {
            w4 = ld8(sm + tl.w + o64);
        } else {
            const uint32_t s2 = tc::pack_bf16x2(sca[128 + r], sca[128 + r]);
            w4 = make_uint2(s2, s2);
        }
        if (PACKED && r >= n) {  // past the sequence (a packed neighbour's tokens): k = q = v = 0
            q4 = make_uint2(0u, 0u);
            k4 = make_uint2(0u, 0u);
            v4 = make_uint2(0u, 0u);
        }
        const uint2 kt4 = (FG2 && fb) ? mul4(k4, sqrt4(b4)) : k4;
        const uint2 kk4 = mul4(kt4, ei4);
        st8(sm + tl.Qp + o128, mul4(q4, e4));                               // Q'
        st8(sm + tl.Kp + o128, mul4(kt4, e4));                              // K'
        st8(sm + tl.Kpp + o128, kk4);                                       // K"
        st8(sm + tl.Bpp + o128, (FG2 && fb) ? kk4 : mul4(b4, kk4));         // B"
        st8(sm + tl.v + o64, mul4((FG2 && fw) ? sqrt4(w4) : w4, v4));       // U
        rev[0] *= bf_lo(apr[xx].x);
        rev[1] *= bf_hi(apr[xx].x);
        rev[2] *= bf_lo(apr[xx].y);
        rev[3] *= bf_hi(apr[xx].y);
    }
    if (q8 == 0 && h == 0) {
        // g_m = gamma_31 (octets 0-3), gc = prod over octets 4-7 (= gamma_63/g_m);
        // the divisors above: prod of a over tokens 1..31 (octet 0 holds it as
        // run * sp) and over tokens 32..63 (gc)
        float gm[4] = {1.f, 1.f, 1.f, 1.f}, gc[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) {
            const float4 qv = *reinterpret_cast<const float4*>(QT + gg * 128 + 4 * cq);
            float* t = gg < 4 ? gm : gc;
            t[0] *= qv.x;
            t[1] *= qv.y;
            t[2] *= qv.z;
            t[3] *= qv.w;
        }
        bool ok = true;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ok = ok && run[j] * pm[j] >= 1e-35f && gc[j] >= 1e-35f;
            chan(4 * cq + j, gm[j], gc[j]);
        }
        if (a_kind != GDR_GATE_ONE && !ok) atomicOr(err_word, kErrRange);
    }
}

// ---------------------------------------------------------------- UT solve
// T = (I + N)^{-1}, N = A_kb strictly lower 64 x 64 (float, row stride NSP, in
// NS), by the 2 x 2 block recursion of a unit lower triangular inverse,
//   [[T1, 0], [T21, T2]] with T21 = -T2 N21 T1,
// applied at 8, 16 and 32 rows: the eight 8 x 8 diagonal inverses by
// substitution and the 8 x 8 blocks below them, then two rounds for the
// 16 x 16 blocks (1,0) and (3,2), then two for the 32 x 32 block below the
// diagonal.  Run by 256 threads (tid 0-255 as passed; barrier id 2).  Each
// finished block also goes, in bf16, into a 64-row operand panel Z3
// (128-byte swizzled rows): T - I + DIAG * I, i.e. T - I for DIAG = 0 and
// T + I for DIAG = 2; the 16 x 16 blocks above the diagonal are not written
// (the caller keeps them zero).

// One element into the 128-byte swizzled Z3 rows.
__device__ __forceinline__ void z3_put(uint8_t* z3, int row, int col, float v) {
    *reinterpret_cast<__nv_bfloat16*>(z3 + row * 128 + (((col >> 3) ^ (row & 7)) << 4) +
                                      2 * (col & 7)) = __float2bfloat16_rn(v);
}
__device__ __forceinline__ void z3_put2(uint8_t* z3, int row, int col, float v0, float v1) {
    *reinterpret_cast<uint32_t*>(z3 + row * 128 + (((col >> 3) ^ (row & 7)) << 4) +
                                 2 * (col & 7)) = tc::pack_bf16x2(v0, v1);
}

// The four 16 x 16 diagonal inverses, themselves by the 2 x 2 recursion at 8
// rows: the eight 8 x 8 diagonal inverses by forward substitution (thread =
// block and column, x_r = [r == c] - sum_{s<r} N_rs x_s), then the 8 x 8
// block below each of their diagonals, T21 = -T2 (N21 T1), one element per
// thread in two steps.  The 8 x 8 block above each diagonal is written zero.
template <int DIAG>
__device__ __forceinline__ void ut_diag(const float* NS, float* TS, float* PS, uint8_t* z3,
                                        int tid) {
    {
        const int B = tid >> 6, r = (tid >> 3) & 7, c = tid & 7;
        TS[(16 * B + r) * NSP + 16 * B + 8 + c] = 0.f;
        z3_put(z3, 16 * B + r, 16 * B + 8 + c, 0.f);
    }
    if (tid < 64) {
        const int I = tid >> 3, c = tid & 7;
        const float* nb = NS + (8 * I) * NSP + 8 * I;
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float acc = (r == c) ? 1.0f : 0.0f;
            if (r > 0) {
                const float4 n0 = *reinterpret_cast<const float4*>(nb + r * NSP);
                const float4 n1 = *reinterpret_cast<const float4*>(nb + r * NSP + 4);
                const float nr[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
#pragma unroll
                for (int s = 0; s < r; ++s) acc = fmaf(-nr[s], x[s], acc);
            }
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            TS[(8 * I + r) * NSP + 8 * I + c] = x[r];
            z3_put(z3, 8 * I + r, 8 * I + c, r > c ? x[r] : (r == c ? (float)DIAG : 0.f));
        }
    }
    half_sync(2);
    const int B = tid >> 6, i = (tid >> 3) & 7, j = tid & 7;
    {
        // P = N21 T1: row i of N21 against column j of T1
        const float* nr = NS + (16 * B + 8 + i) * NSP + 16 * B;
        const float* tc = TS + (16 * B) * NSP + 16 * B + j;
        const float4 n0 = *reinterpret_cast<const float4*>(nr);
        const float4 n1 = *reinterpret_cast<const float4*>(nr + 4);
        const float nv[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
        float p = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) p = fmaf(nv[k], tc[k * NSP], p);
        PS[64 * B + 8 * i + j] = p;
    }
    half_sync(2);
    {
        // T21 = -T2 P: row i of T2 against column j of P
        const float* tr = TS + (16 * B + 8 + i) * NSP + 16 * B + 8;
        const float4 t0 = *reinterpret_cast<const float4*>(tr);
        const float4 t1 = *reinterpret_cast<const float4*>(tr + 4);
        const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
        const float* pc = PS + 64 * B + j;
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) v = fmaf(tv[k], pc[8 * k], v);
        TS[(16 * B + 8 + i) * NSP + 16 * B + j] = -v;
        z3_put(z3, 16 * B + 8 + i, 16 * B + j, -v);
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
    ut_diag<DIAG>(NS, TS, PS, z3, tid);
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
