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
//   E  = T (Kh S0 + A_kk U),             Kh = gamma*K   (row r: S'_r^T k_r)
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
// the grams are [K';Q'] [K";B"]^T, and with the state kept as
// S~ = Diag(g_m) S0 the same four tiles serve every other product:
//   E^T  = S~^T (T K')^T + (A_kk U)^T T^T
//   O^T  = S~^T Q'^T + U^T A_qk^T - E^T A_qb^T
//   S~^T <- S~^T + U^T K" - E^T B"      then S_new = Diag(gamma_C/g_m) S~.
// Every factor is exp of the decay accumulated over at most half a chunk.  If
// that exceeds exp(80) in some channel the factors leave float range; the
// kernel then sets GDR_ERR_RANGE in the device error word (the float32
// CUDA-core kernel, chunk <= 32, has no such limit).
//
// State-side products are formed transposed so that every product has
// M = 128 (tensor-memory lane = value channel j).  S~^T stays in float32 in
// tensor memory for the whole sequence; a bf16 copy in shared memory is the
// MMA operand.  One CTA (16 warps) owns one (batch, head) and walks its
// chunks in order.  Raw q/k/v and vector gates arrive by TMA as 64-token x
// 64-channel boxes, 128-byte swizzled, i.e. already in the operand layout of
// tc_common.cuh; the next chunk's q and k are fetched while the current one
// is processed, and o leaves by a TMA store.  Products are tcgen05.mma issued
// by one thread; the cumulative decay, the UT solve and the conversions run
// on the CUDA cores with 16-byte shared-memory accesses.
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
constexpr uint32_t OFF_X1 = 32768;      // [K'; Q'] 128 rows x 128; o staging at the end
constexpr uint32_t OFF_X2 = 65536;      // [K"; B"] 128 rows x 128 (raw a, b land here)
constexpr uint32_t OFF_U = 98304;       // U = w*v [s][j] (raw v lands here)
constexpr uint32_t OFF_L = 114688;      // A_kk strictly lower [r][s] (raw w lands at L..AQK)
constexpr uint32_t OFF_AQK = 122880;    // A_qk lower [r][s]
constexpr uint32_t OFF_AQB = 131072;    // -A_qb lower [r][s]
constexpr uint32_t OFF_T = 139264;      // T [r][s] bf16
constexpr uint32_t OFF_S0T = 147456;    // S~^T [j][i] bf16, 2 panels
constexpr uint32_t OFF_R = 180224;      // scratch region, 36 KB:
constexpr uint32_t OFF_REL = OFF_R;             //  P1: log(gamma_r) partial sums, float [64][128]
constexpr uint32_t OFF_QT = OFF_R + 32768;      //  P1: quarter totals, float [4][128]
constexpr uint32_t OFF_OFS = OFF_R + 34816;     //  P1: per-quarter offsets, float [4][128]
constexpr uint32_t OFF_NS = OFF_R;              //  P4-P5: A_kb, float [64][65]
constexpr uint32_t OFF_TS = OFF_R + 16640;      //  P5: T, float [64][65]
constexpr uint32_t OFF_PS = OFF_R + 33280;      //  P5: float [3][256]
constexpr uint32_t OFF_W = OFF_R;               //  P7-P8: (T K')^T [i][r]
constexpr uint32_t OFF_ZT = OFF_R + 16384;      //  P7-P8: (A_kk U)^T [j][s]
constexpr uint32_t OFF_ET = OFF_R;              //  P9-P10: E^T [j][r]
constexpr uint32_t OFF_SMALL = OFF_R + 36864;   // 217088
constexpr uint32_t OFF_FCUR = OFF_SMALL;        // float[128]: state scale this chunk
constexpr uint32_t OFF_FPREV = OFF_SMALL + 512; // float[128]: gamma_C/g_m of last chunk
constexpr uint32_t OFF_SCA = OFF_SMALL + 1024;  // float[3][64]: scalar a, b, w
constexpr uint32_t OFF_BAR = OFF_SMALL + 1792;  // 3 mbarriers: mma, kq, rest
constexpr uint32_t OFF_TSLOT = OFF_BAR + 24;
constexpr uint32_t OFF_ABORT = OFF_BAR + 28;
constexpr uint32_t SMEM_USED = OFF_BAR + 32;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");

constexpr int NSP = 65;  // row stride (floats) of the solve's float tiles

// ---- tensor-memory columns (512 allocated)
constexpr uint32_t TM_G = 0;     // gram 128 x 128
constexpr uint32_t TM_W = 128;   // (T K')^T 128 x 64
constexpr uint32_t TM_Z = 192;   // (A_kk U)^T 128 x 64
constexpr uint32_t TM_E = 256;   // E^T  128 x 64
constexpr uint32_t TM_O = 320;   // O^T  128 x 64
constexpr uint32_t TM_S = 384;   // S~^T 128 x 128, float32 state

constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr uint32_t BOX_BYTES = 64 * 128;     // one 64 x 64 bf16 TMA box
constexpr uint32_t IDESC_NEG_B = 1u << 14;   // negate the B operand

struct TcMaps {
    CUtensorMap q, k, v, a, b, w, o;  // a/b/w only meaningful for vector gates
};

__device__ __forceinline__ float ld_bf16_sm(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// 8 bf16 (one 16-byte chunk) <-> 8 floats
__device__ __forceinline__ void unpack8(uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        f[2 * x] = __uint_as_float(w[x] << 16);
        f[2 * x + 1] = __uint_as_float(w[x] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    u.x = tc::pack_bf16x2(f[0], f[1]);
    u.y = tc::pack_bf16x2(f[2], f[3]);
    u.z = tc::pack_bf16x2(f[4], f[5]);
    u.w = tc::pack_bf16x2(f[6], f[7]);
    return u;
}

// ---------------------------------------------------------------- UT solve
// T = (I + N)^{-1}, N strictly lower 64 x 64 in NS, T into TS (both float,
// row stride NSP).  The four 16 x 16 diagonal blocks by right-looking
// substitution, then the off-diagonal blocks level by level:
//   T_IJ = -T_II * P,  P = sum_{s in blocks J..I-1} N[I rows][s] T[s][J cols].
template <int LVL>
__device__ __forceinline__ void ut_level(const float* NS, float* TS, float* PS, int tid) {
    constexpr int NB = 4 - LVL;
    for (int x = tid; x < NB * 256; x += NT) {
        const int b = x >> 8, e = x & 255, rho = e >> 4, kap = e & 15;
        const int I = LVL + b, J = b;
        const float* nr = NS + (16 * I + rho) * NSP + 16 * J;
        const float* tc_ = TS + (16 * J) * NSP + 16 * J + kap;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 16 * LVL; ++s) acc[s & 3] = fmaf(nr[s], tc_[s * NSP], acc[s & 3]);
        PS[x] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
    for (int x = tid; x < NB * 256; x += NT) {
        const int b = x >> 8, e = x & 255, rho = e >> 4, kap = e & 15;
        const int I = LVL + b, J = b;
        const float* tr = TS + (16 * I + rho) * NSP + 16 * I;  // row of T_II (zero above diag)
        const float* pc = PS + (b << 8) + kap;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int sg = 0; sg < 16; ++sg) acc[sg & 3] = fmaf(tr[sg], pc[sg << 4], acc[sg & 3]);
        TS[(16 * I + rho) * NSP + 16 * J + kap] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
    __syncthreads();
}

__device__ void ut_solve(const float* NS, float* TS, float* PS, int tid) {
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
    __syncthreads();
    ut_level<1>(NS, TS, PS, tid);
    ut_level<2>(NS, TS, PS, tid);
    ut_level<3>(NS, TS, PS, tid);
}

// ---------------------------------------------------------------- TMA issue
// Group "kq": raw k and q into the RAW tile.  Group "rest": vector a and b
// into X2, v into U, vector w into L..AQK.
__device__ __forceinline__ void issue_kq(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                         uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 4 * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384, &m.k, 64 * p, hi, t0, bi, bar);
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384 + 8192, &m.q, 64 * p, hi, t0, bi, bar);
    }
}

__device__ __forceinline__ void issue_rest(const TcMaps& m, uint32_t sbase, int t0, int hi,
                                           int bi, bool va, bool vb, bool vw, uint32_t bar) {
    const uint32_t nbox = 2u * (1u + (va ? 1u : 0u) + (vb ? 1u : 0u) + (vw ? 1u : 0u));
    tc::mbar_arrive_expect_tx(bar, nbox * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        tc::tma_load_4d(sbase + OFF_U + p * 8192, &m.v, 64 * p, hi, t0, bi, bar);
        if (va) tc::tma_load_4d(sbase + OFF_X2 + p * 16384, &m.a, 64 * p, hi, t0, bi, bar);
        if (vb) tc::tma_load_4d(sbase + OFF_X2 + p * 16384 + 8192, &m.b, 64 * p, hi, t0, bi, bar);
        if (vw) tc::tma_load_4d(sbase + OFF_L + p * 8192, &m.w, 64 * p, hi, t0, bi, bar);
    }
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
    float* REL = reinterpret_cast<float*>(sm + OFF_REL);
    float* QT = reinterpret_cast<float*>(sm + OFF_QT);
    float* OFS = reinterpret_cast<float*>(sm + OFF_OFS);
    float* NS = reinterpret_cast<float*>(sm + OFF_NS);
    float* TS = reinterpret_cast<float*>(sm + OFF_TS);
    float* PS = reinterpret_cast<float*>(sm + OFF_PS);
    float* fcur = reinterpret_cast<float*>(sm + OFF_FCUR);
    float* fprev = reinterpret_cast<float*>(sm + OFF_FPREV);
    float* sca = reinterpret_cast<float*>(sm + OFF_SCA);
    volatile int* abort_s = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
    const uint32_t bar_mma = sbase + OFF_BAR;
    const uint32_t bar_kq = sbase + OFF_BAR + 8;
    const uint32_t bar_rs = sbase + OFF_BAR + 16;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quarter = warp & 3;               // tensor-memory lanes 32*quarter ..
    const int cb = warp >> 2;                   // 32-column block this warp reads
    const int lane_j = 32 * quarter + (tid & 31);  // tensor-memory lane of this thread
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;

    const int bh = blockIdx.x;
    const int bi = bh / H, hi = bh % H;
    const size_t soff = (size_t)bh * D * D;
    const bool va = a_kind == GDR_GATE_VECTOR, vb = b_kind == GDR_GATE_VECTOR,
               vw = w_kind == GDR_GATE_VECTOR;

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_kq, 1);
        tc::mbar_init(bar_rs, 1);
        tc::mbar_fence_init();
        *abort_s = 0;
        tc::tma_prefetch_desc(&maps.q);
        tc::tma_prefetch_desc(&maps.k);
        tc::tma_prefetch_desc(&maps.v);
        tc::tma_prefetch_desc(&maps.o);
    }
    if (tid < D) fprev[tid] = 1.0f;
    if (warp == 0) tc::tmem_alloc(sbase + OFF_TSLOT, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TSLOT);
    uint32_t ph_mma = 0, ph_kq = 0, ph_rs = 0;

    if (tid == 0 && T > 0) {
        issue_kq(maps, sbase, 0, hi, bi, bar_kq);
        issue_rest(maps, sbase, 0, hi, bi, va, vb, vw, bar_rs);
    }
    // scalar gates of the next chunk, loaded a chunk ahead
    float a_nx = 1.f, b_nx = 1.f, w_nx = 1.f;
    auto load_scalars = [&](int t0n) {
        if (tid < C) {
            const int nn = min(C, T - t0n);
            const long long tok = ((long long)bi * T + t0n + tid) * H + hi;
            const bool in = tid < nn;
            a_nx = (a_kind == GDR_GATE_SCALAR && in) ? to_f32(a[tok]) : 1.f;
            b_nx = (b_kind == GDR_GATE_SCALAR && in) ? to_f32(b[tok]) : 1.f;
            w_nx = (w_kind == GDR_GATE_SCALAR && in) ? to_f32(w[tok]) : 1.f;
        }
    };
    if (T > 0) load_scalars(0);

    // ---- initial state S0^T (unscaled) into tensor memory
    {
        const int c0 = 32 * cb;
        float vals[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) vals[x] = s0 ? s0[soff + (size_t)(c0 + x) * D + lane_j] : 0.0f;
        tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
        tc::tmem_wait_st();
    }
    tc::fence_before_sync();
    __syncthreads();

#pragma unroll 1
    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        const bool has_next = t0 + C < T;

        // ================= P1: wait for the chunk, cumulative decay, operands
        if (tid < C) {
            sca[tid] = a_nx;
            sca[64 + tid] = b_nx;
            sca[128 + tid] = w_nx;
        }
        if (tid == 0) tc::bulk_wait_read();  // the previous o store has left X1
        if (!tc::mbar_wait_bounded(bar_kq, ph_kq, WAIT_NS)) *abort_s = 1;
        if (!tc::mbar_wait_bounded(bar_rs, ph_rs, WAIT_NS)) *abort_s = 1;
        ph_kq ^= 1;
        ph_rs ^= 1;
        __syncthreads();
        {
            // pass A: log-decay partial sums over 16-token quarters, channel i
            const int i = tid & 127, qr = tid >> 7;
            const int pch = i >> 6, cc = i & 63;
            const uint32_t colb = ((uint32_t)(cc & 7) << 1);
            const int chunk8 = cc >> 3;
            float run = 0.f, first = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int r = 16 * qr + u;
                float g = 0.f;
                if (a_kind != GDR_GATE_ONE && r < n) {
                    const float av =
                        va ? ld_bf16_sm(sm + OFF_X2, (uint32_t)pch * 16384u + (uint32_t)r * 128u +
                                                         ((uint32_t)(chunk8 ^ (r & 7)) << 4) + colb)
                           : sca[r];
                    g = safe_log_decay(av);
                }
                run += g;
                if (u == 0) first = run;
                REL[r * D + i] = run;
            }
            QT[qr * D + i] = run;
            __syncthreads();
            // pass B: per-quarter offsets so that REL + OFS = log(gamma_r / g_m)
            const float q0 = QT[i], q1 = QT[D + i], q2 = QT[2 * D + i], q3 = QT[3 * D + i];
            const float T0 = q0 + q1, T1 = q2 + q3;
            const float pre = (qr > 0 ? q0 : 0.f) + (qr > 1 ? q1 : 0.f) + (qr > 2 ? q2 : 0.f);
            OFS[qr * D + i] = pre - T0;
            if (qr == 0) {
                fcur[i] = fprev[i] * __expf(T0);   // scale of S~ this chunk
                fprev[i] = __expf(T1);             // gamma_C / g_m, applied next chunk
                if (a_kind != GDR_GATE_ONE && (first - T0 > 80.f || T1 < -80.f))
                    atomicOr(err_word, kErrRange);
            }
            __syncthreads();
            // pass C: scaled operands, 8 channels (16 bytes) per access
#pragma unroll 1
            for (int it = tid; it < C * 16; it += NT) {
                const int r = it >> 4, c16 = it & 15, p = c16 >> 3, ch = c16 & 7;
                const uint32_t swz = ((uint32_t)(ch ^ (r & 7)) << 4) + (uint32_t)r * 128u;
                const uint32_t otop = (uint32_t)p * 16384u + swz;  // rows 0-63 of 128-row tiles
                const uint32_t obot = otop + 8192u;                // rows 64-127
                const uint32_t o64 = (uint32_t)p * 8192u + swz;    // 64-row tiles
                float kf[8], qf[8], bf[8], vf[8], wf[8], rel[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + OFF_RAW + otop), kf);
                unpack8(*reinterpret_cast<const uint4*>(sm + OFF_RAW + obot), qf);
                unpack8(*reinterpret_cast<const uint4*>(sm + OFF_U + o64), vf);
                if (vb) {
                    unpack8(*reinterpret_cast<const uint4*>(sm + OFF_X2 + obot), bf);
                } else {
#pragma unroll
                    for (int x = 0; x < 8; ++x) bf[x] = sca[64 + r];
                }
                if (vw) {
                    unpack8(*reinterpret_cast<const uint4*>(sm + OFF_L + o64), wf);
                } else {
#pragma unroll
                    for (int x = 0; x < 8; ++x) wf[x] = sca[128 + r];
                }
                const float4* rp = reinterpret_cast<const float4*>(REL + r * D + 8 * c16);
                const float4* op = reinterpret_cast<const float4*>(OFS + (r >> 4) * D + 8 * c16);
                const float4 r0 = rp[0], r1 = rp[1], f0 = op[0], f1 = op[1];
                rel[0] = r0.x + f0.x; rel[1] = r0.y + f0.y; rel[2] = r0.z + f0.z; rel[3] = r0.w + f0.w;
                rel[4] = r1.x + f1.x; rel[5] = r1.y + f1.y; rel[6] = r1.z + f1.z; rel[7] = r1.w + f1.w;
                float o1[8], o2[8], o3[8], o4[8], o5[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float e1 = __expf(rel[x]);
                    const float e1i = __expf(-rel[x]);
                    o1[x] = kf[x] * e1;
                    o2[x] = qf[x] * e1;
                    o3[x] = kf[x] * e1i;
                    o4[x] = bf[x] * kf[x] * e1i;
                    o5[x] = wf[x] * vf[x];
                }
                *reinterpret_cast<uint4*>(sm + OFF_X1 + otop) = pack8(o1);
                *reinterpret_cast<uint4*>(sm + OFF_X1 + obot) = pack8(o2);
                *reinterpret_cast<uint4*>(sm + OFF_X2 + otop) = pack8(o3);
                *reinterpret_cast<uint4*>(sm + OFF_X2 + obot) = pack8(o4);
                *reinterpret_cast<uint4*>(sm + OFF_U + o64) = pack8(o5);
            }
        }
        tc::fence_async_smem();
        __syncthreads();
        if (*abort_s) break;
        // the RAW tile is free: fetch the next chunk's k and q now
        if (tid == 0 && has_next) issue_kq(maps, sbase, t0 + C, hi, bi, bar_kq);

        // ================= P2: S~^T <- S~^T * f (column i), bf16 copy to smem
        tc::fence_after_sync();
        {
            const int c0 = 32 * cb;
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
            tc::tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) vals[x] *= fcur[c0 + x];
            tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
            tc::store_row32_bf16(sm + OFF_S0T + (cb >> 1) * 16384, lane_j, cb & 1, vals);
            tc::tmem_wait_st();
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // ================= P3: gram [K';Q'] [K";B"]^T
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_G, tc::desc_kmajor(sbase + OFF_X1, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_X2, 16384, kk), id, kk > 0);
            tc::mma_commit(bar_mma);
        }
        if (!tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS)) *abort_s = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();

        // ================= P4: read the gram; masked blocks out
        {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_G + 32 * cb, vals);
            tc::tmem_wait_ld();
            const bool top = lane_j < 64;  // rows of K' (else Q')
            const int r = top ? lane_j : lane_j - 64;
            const int s0c = 32 * (cb & 1);  // first s of this column block
            if (cb < 2) {
                // A_kk (strictly lower) or A_qk (lower incl. diagonal)
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    vals[x] = (top ? (s0c + x < r) : (s0c + x <= r)) ? vals[x] : 0.f;
                tc::store_row32_bf16(sm + (top ? OFF_L : OFF_AQK), r, cb & 1, vals);
            } else if (top) {
                float* nrow = NS + r * NSP + s0c;
#pragma unroll
                for (int x = 0; x < 32; ++x) nrow[x] = (s0c + x < r) ? vals[x] : 0.f;
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] = (s0c + x <= r) ? -vals[x] : 0.f;
                tc::store_row32_bf16(sm + OFF_AQB, r, cb & 1, vals);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        if (*abort_s) break;

        // ================= P5: UT transform T = (I + A_kb)^{-1}
        ut_solve(NS, TS, PS, tid);
        {
            const int r = tid >> 3, ch = tid & 7;  // 64 rows x 8 chunks of 8
            float vals[8];
            const float* trow = TS + r * NSP + 8 * ch;
#pragma unroll
            for (int x = 0; x < 8; ++x) vals[x] = (8 * ch + x <= r) ? trow[x] : 0.f;
            *reinterpret_cast<uint4*>(sm + OFF_T + r * 128 + ((ch ^ (r & 7)) << 4)) = pack8(vals);
        }
        tc::fence_async_smem();
        __syncthreads();

        // ================= P6: (T K')^T = K'^T T^T and (A_kk U)^T = U^T A_kk^T
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id = tc::idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                tc::mma_bf16(tmem + TM_W, tc::desc_mnmajor(sbase + OFF_X1, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_T, 8192, kk), id, kk > 0);
                tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_kmajor(sbase + OFF_L, 8192, kk), id, kk > 0);
            }
            tc::mma_commit(bar_mma);
        }
        if (!tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS)) *abort_s = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();

        // ================= P7: (T K')^T -> smem [i][r], (A_kk U)^T -> smem [j][s]
        {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_W + 32 * cb, vals);  // TM_Z = TM_W + 64
            tc::tmem_wait_ld();
            tc::store_row32_bf16(sm + (cb < 2 ? OFF_W : OFF_ZT), lane_j, cb & 1, vals);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // ================= P8: E^T = S~^T (T K')^T + (A_kk U)^T T^T
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id1 = tc::idesc_bf16(128, 64, 0, 1);
            const uint32_t id2 = tc::idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_E, tc::desc_kmajor(sbase + OFF_S0T, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_W, 16384, kk), id1, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_E, tc::desc_kmajor(sbase + OFF_ZT, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_T, 8192, kk), id2, true);
            tc::mma_commit(bar_mma);
        }
        if (!tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS)) *abort_s = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();

        // ================= P9: E^T -> smem [j][r]
        if (cb < 2) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_E + 32 * cb, vals);
            tc::tmem_wait_ld();
            tc::store_row32_bf16(sm + OFF_ET, lane_j, cb, vals);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // ================= P10: O^T and the state update
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idKK = tc::idesc_bf16(128, 64, 0, 0);
            const uint32_t idMK = tc::idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_bf16(tmem + TM_O, tc::desc_kmajor(sbase + OFF_S0T, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_X1 + 8192, 16384, kk), idKK, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_O, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_kmajor(sbase + OFF_AQK, 8192, kk), idMK, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_O, tc::desc_kmajor(sbase + OFF_ET, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_AQB, 8192, kk), idKK, true);
            const uint32_t idMM = tc::idesc_bf16(128, 128, 1, 1);
            const uint32_t idKMn = tc::idesc_bf16(128, 128, 0, 1) | IDESC_NEG_B;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_mnmajor(sbase + OFF_X2, 16384, kk), idMM, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_kmajor(sbase + OFF_ET, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_X2 + 8192, 16384, kk), idKMn, true);
            tc::mma_commit(bar_mma);
        }
        if (!tc::mbar_wait_bounded(bar_mma, ph_mma, WAIT_NS)) *abort_s = 1;
        ph_mma ^= 1;
        tc::fence_after_sync();
        // X2, U, L..AQK are free: fetch the next chunk's v and vector gates
        if (tid == 0 && has_next) issue_rest(maps, sbase, t0 + C, hi, bi, va, vb, vw, bar_rs);
        if (has_next) load_scalars(t0 + C);

        // ================= P11: O^T -> [token][channel] tile in X1 -> TMA store
        if (cb < 2) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_O + 32 * cb, vals);
            tc::tmem_wait_ld();
            const int j = lane_j, pj = j >> 6, cj = j & 63;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const int r = 32 * cb + x;
                const uint32_t off = (uint32_t)pj * 8192u + (uint32_t)r * 128u +
                                     ((uint32_t)(((cj >> 3) ^ (r & 7))) << 4) +
                                     ((uint32_t)(cj & 7) << 1);
                *reinterpret_cast<__nv_bfloat16*>(sm + OFF_X1 + off) = __float2bfloat16_rn(vals[x]);
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_4d(&maps.o, sbase + OFF_X1, 0, hi, t0, bi);
            tc::tma_store_4d(&maps.o, sbase + OFF_X1 + 8192, 64, hi, t0, bi);
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
            tc::mbar_wait_bounded(bar_rs, ph_rs, WAIT_NS);
        }
        __syncthreads();
    } else if (s_final) {
        tc::fence_after_sync();
        const int c0 = 32 * cb;
        float vals[32];
        tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
        tc::tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x)
            s_final[soff + (size_t)(c0 + x) * D + lane_j] = vals[x] * fprev[c0 + x];
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
