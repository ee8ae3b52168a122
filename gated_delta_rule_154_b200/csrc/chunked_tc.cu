// chunked_tc.cu -- chunkwise-parallel gated delta rule on the Blackwell
// tensor cores (tcgen05, accumulators in tensor memory), bf16 inputs,
// float32 state, dk = dv = 128, chunk C = 64.
//
// Chunked form (per chunk of n <= 64 tokens, state S0 at its start,
// gamma_r = prod_{i<=r} a_i per key channel, U = w*V, m = token 31):
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
// Grams use the factorisation gamma_r/gamma_s = (gamma_r/gamma_m)(gamma_m/gamma_s)
// around the chunk's middle token m, so every factor is exp of the decay
// accumulated over at most half a chunk.  If that exceeds exp(80) in some
// channel the factors leave float range; the kernel then sets GDR_ERR_RANGE
// in the device error word (the float32 CUDA-core kernel, chunk <= 32, has no
// such limit).
//
// Everything state-side is computed transposed so that every product has
// M = 128 on the tensor core (lanes of tensor memory = value channel j):
//   E^T   = S0^T W^T + Z^T T^T          W = T Kh, Z = A_kk U
//   O^T   = S0^T Qh^T + U^T A_qk^T - E^T A_qb^T
//   S^T  += U^T Kt - E^T Bt             (S^T kept in float32 in tensor memory,
//                                        pre-scaled by gamma_C)
// One CTA (256 threads) owns one (batch, head) and walks its chunks in order.
// Products run on tcgen05.mma issued by one thread; the UT solve, the gate
// arithmetic and the conversions run on the CUDA cores.  Operands are bf16
// in shared memory in the swizzled row format of tc_common.cuh.
#include "common.cuh"
#include "tc_common.cuh"

namespace gdr {
namespace {

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // dk = dv
constexpr int NT = 256;      // threads per CTA

// ---- shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_X1 = 0;          // [K'; Q'] 128 rows x 128, gram A operand
constexpr uint32_t OFF_X2 = 32768;      // [K"; B"] 128 rows x 128, gram B operand
constexpr uint32_t OFF_W = 0;           // W^T  [i][r]  (aliases X1 after the gram)
constexpr uint32_t OFF_ZT = 16384;      // Z^T  [j][s]  (aliases X1)
constexpr uint32_t OFF_NS = 32768;      // A_kb strictly lower, float [64][65] (aliases X2)
constexpr uint32_t OFF_TS = 49408;      // T, float [64][65]
constexpr uint32_t OFF_PS = 66048;      // solve scratch, float [3][256]
constexpr uint32_t OFF_KH = 69632;      // Kh  [s][i]
constexpr uint32_t OFF_ET = 69632;      // E^T [j][r] (aliases Kh after W is formed)
constexpr uint32_t OFF_QH = 86016;      // Qh  [r][i]
constexpr uint32_t OFF_U = 102400;      // U   [s][j]
constexpr uint32_t OFF_KT = 118784;     // Kt  [s][i]
constexpr uint32_t OFF_BT = 135168;     // -Bt [s][i]
constexpr uint32_t OFF_L = 151552;      // A_kk strictly lower [r][s]
constexpr uint32_t OFF_AQK = 159744;    // A_qk lower [r][s]
constexpr uint32_t OFF_AQB = 167936;    // -A_qb lower [r][s]
constexpr uint32_t OFF_T = 176128;      // T [r][s] bf16
constexpr uint32_t OFF_S0T = 184320;    // S0^T [j][i] bf16, 2 panels
constexpr uint32_t OFF_GC = 217088;     // gamma_C per key channel, float[128]
constexpr uint32_t OFF_BAR = 217600;    // mbarrier
constexpr uint32_t OFF_TSLOT = 217608;  // tensor-memory base address
constexpr uint32_t OFF_ABORT = 217612;  // set when a wait ran out
constexpr uint32_t SMEM_USED = 217616;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

constexpr int NSP = 65;  // row stride (floats) of the solve's float tiles

// ---- tensor-memory columns (512 allocated)
constexpr uint32_t TM_G = 0;     // gram 128 x 128
constexpr uint32_t TM_W = 128;   // W^T  128 x 64
constexpr uint32_t TM_Z = 192;   // Z^T  128 x 64
constexpr uint32_t TM_E = 256;   // E^T  128 x 64
constexpr uint32_t TM_O = 320;   // O^T  128 x 64
constexpr uint32_t TM_S = 384;   // S^T  128 x 128, float32 state

constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per tensor-core wait

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float v) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(v);
}

template <typename Tin>
__device__ __forceinline__ float ldg_f(const Tin* p) {
    return to_f32(__ldg(p));
}

// Forward substitution for T = (I + N)^{-1}, N strictly lower 64 x 64 in NS,
// T written to TS (both float, row stride NSP).  Blocked: the four 16 x 16
// diagonal blocks by substitution, then the off-diagonal blocks level by
// level, T_IJ = -T_II * sum_{s in blocks J..I-1} N[I rows][s] T[s][J cols].
__device__ void ut_solve(const float* NS, float* TS, float* PS, int tid) {
    if (tid < 64) {
        const int I = tid >> 4, c = tid & 15, col = 16 * I + c;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == c) ? 1.0f : 0.0f;
            const float* nr = NS + (16 * I + r) * NSP + 16 * I;
#pragma unroll
            for (int s = 0; s < r; ++s) acc = fmaf(-nr[s], x[s], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) TS[(16 * I + r) * NSP + col] = x[r];
    }
    __syncthreads();
#pragma unroll 1
    for (int lvl = 1; lvl < 4; ++lvl) {
        const int nb = 4 - lvl;
        for (int x = tid; x < nb * 256; x += NT) {
            const int b = x >> 8, e = x & 255, rho = e >> 4, kap = e & 15;
            const int I = lvl + b, J = b;
            const float* nr = NS + (16 * I + rho) * NSP;
            float acc = 0.f;
            for (int s = 16 * J; s < 16 * I; ++s) acc = fmaf(nr[s], TS[s * NSP + 16 * J + kap], acc);
            PS[x] = acc;
        }
        __syncthreads();
        for (int x = tid; x < nb * 256; x += NT) {
            const int b = x >> 8, e = x & 255, rho = e >> 4, kap = e & 15;
            const int I = lvl + b, J = b;
            const float* tr = TS + (16 * I + rho) * NSP + 16 * I;
            float acc = 0.f;
            for (int sg = 0; sg <= rho; ++sg) acc = fmaf(tr[sg], PS[(b << 8) + (sg << 4) + kap], acc);
            TS[(16 * I + rho) * NSP + 16 * J + kap] = -acc;
        }
        __syncthreads();
    }
}

template <typename Tin>
__global__ void __launch_bounds__(NT, 1)
chunked_tc_kernel(int B, int T, int H, const Tin* __restrict__ q, const Tin* __restrict__ k,
                  const Tin* __restrict__ v, const Tin* __restrict__ a,
                  const Tin* __restrict__ b, const Tin* __restrict__ w, int a_kind,
                  int b_kind, int w_kind, const float* __restrict__ s0, Tin* __restrict__ o,
                  float* __restrict__ s_final, int* __restrict__ err_word) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float* NS = reinterpret_cast<float*>(sm + OFF_NS);
    float* TS = reinterpret_cast<float*>(sm + OFF_TS);
    float* PS = reinterpret_cast<float*>(sm + OFF_PS);
    float* gC_s = reinterpret_cast<float*>(sm + OFF_GC);
    volatile int* abort_s = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
    const uint32_t bar = sbase + OFF_BAR;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int grp = tid >> 7;         // 0: warps 0-3, 1: warps 4-7
    const int gl = tid & 127;         // tensor-memory lane / channel of this thread
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;

    const int bh = blockIdx.x;
    const int bi = bh / H, hi = bh % H;
    const size_t soff = (size_t)bh * D * D;

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
        *abort_s = 0;
    }
    if (warp == 0) tc::tmem_alloc(sbase + OFF_TSLOT, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TSLOT);
    uint32_t phase = 0;

    // ---- initial state: S^T into tensor memory (float) and S0^T (bf16) into smem
    if (grp == 1) {
        const int j = gl;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            float vals[32];
#pragma unroll
            for (int x = 0; x < 32; ++x)
                vals[x] = s0 ? s0[soff + (size_t)(c0 + x) * D + j] : 0.0f;
            tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
            tc::store_row32_bf16(sm + OFF_S0T + (c0 >> 6) * 16384, j, (c0 >> 5) & 1, vals);
        }
        tc::tmem_wait_st();
    }
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    const long long row_stride = (long long)H;  // tokens are H rows apart in [B,T,H,*]
#pragma unroll 1
    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        const long long tok0 = ((long long)bi * T + t0) * H + hi;

        // ================= P1: gates, cumulative decay, scaled operands
        {
            const int i = gl;
            float Gh[32];
            float Gm = 0.f, run = 0.f;
#pragma unroll
            for (int r = 0; r < C; ++r) {
                float g = 0.f;
                if (a_kind != GDR_GATE_ONE && r < n) {
                    const long long tok = tok0 + r * row_stride;
                    const float av = (a_kind == GDR_GATE_SCALAR) ? ldg_f(a + tok)
                                                                 : ldg_f(a + tok * D + i);
                    g = safe_log_decay(av);
                }
                run += g;
                if (r < 32) {
                    if (grp == 0) Gh[r] = run;
                } else {
                    if (grp == 1) Gh[r - 32] = run;
                }
                if (r == 31) Gm = run;
            }
            const float GC = run;
            if (grp == 0) {
                gC_s[i] = __expf(GC);
                if (a_kind != GDR_GATE_ONE && (Gh[0] - Gm > 80.f || Gm - GC > 80.f))
                    atomicOr(err_word, kErrRange);
            }
            const float eGm = __expf(Gm);
            const float eCm = __expf(GC - Gm);
            const int pch = i >> 6, cc = i & 63;
            const uint32_t colb = ((uint32_t)(cc & 7) << 1);
            const int chunk8 = cc >> 3;
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) {
                const int r = 32 * grp + rr;
                float kv = 0.f, qv = 0.f, bv = 0.f, uv = 0.f;
                if (r < n) {
                    const long long tok = tok0 + r * row_stride;
                    kv = ldg_f(k + tok * D + i);
                    qv = ldg_f(q + tok * D + i);
                    bv = (b_kind == GDR_GATE_ONE) ? 1.f
                         : (b_kind == GDR_GATE_SCALAR) ? ldg_f(b + tok) : ldg_f(b + tok * D + i);
                    const float wv = (w_kind == GDR_GATE_ONE) ? 1.f
                                     : (w_kind == GDR_GATE_SCALAR) ? ldg_f(w + tok)
                                                                   : ldg_f(w + tok * D + i);
                    uv = wv * ldg_f(v + tok * D + i);
                }
                const float e1 = __expf(Gh[rr] - Gm);     // gamma_r / gamma_m
                const float e1i = 1.0f / e1;               // gamma_m / gamma_r
                const float eg = e1 * eGm;                 // gamma_r
                const float et = eCm * e1i;                // gamma_C / gamma_r
                const float bk = bv * kv;
                const uint32_t sw = ((uint32_t)(chunk8 ^ (r & 7)) << 4) + colb;
                // 128-row tiles (panel 16 KB) and 64-row tiles (panel 8 KB)
                const uint32_t o128a = (uint32_t)pch * 16384u + (uint32_t)r * 128u + sw;
                const uint32_t o128b = o128a + 64u * 128u;
                const uint32_t o64 = (uint32_t)pch * 8192u + (uint32_t)r * 128u + sw;
                st_bf16(sm + OFF_X1, o128a, kv * e1);
                st_bf16(sm + OFF_X1, o128b, qv * e1);
                st_bf16(sm + OFF_X2, o128a, kv * e1i);
                st_bf16(sm + OFF_X2, o128b, bk * e1i);
                st_bf16(sm + OFF_KH, o64, kv * eg);
                st_bf16(sm + OFF_QH, o64, qv * eg);
                st_bf16(sm + OFF_KT, o64, kv * et);
                st_bf16(sm + OFF_BT, o64, -bk * et);
                st_bf16(sm + OFF_U, o64, uv);
            }
        }
        __syncthreads();

        // ================= P2: S^T <- S^T * gamma_C (column i scaled)
        tc::fence_after_sync();
        {
#pragma unroll 1
            for (int c0 = 64 * grp; c0 < 64 * grp + 64; c0 += 32) {
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
                tc::tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] *= gC_s[c0 + x];
                tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
            }
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
            tc::mma_commit(bar);
        }
        if (!tc::mbar_wait_bounded(bar, phase, WAIT_NS)) *abort_s = 1;
        phase ^= 1;
        tc::fence_after_sync();

        // ================= P4: read the gram; masked blocks out
        {
            float vals[64];
            tc::tmem_ld32(tmem + lane_off + TM_G + 64 * grp, vals);
            tc::tmem_ld32(tmem + lane_off + TM_G + 64 * grp + 32, vals + 32);
            tc::tmem_wait_ld();
            const bool top = gl < 64;  // rows of K' (else Q')
            const int r = top ? gl : gl - 64;
            if (grp == 0) {
                // A_kk (strictly lower) or A_qk (lower incl. diagonal)
#pragma unroll
                for (int s = 0; s < 64; ++s)
                    vals[s] = (top ? (s < r) : (s <= r)) ? vals[s] : 0.f;
                tc::store_row64_bf16(sm + (top ? OFF_L : OFF_AQK), r, vals);
            } else if (top) {
                float* nrow = NS + r * NSP;
#pragma unroll
                for (int s = 0; s < 64; ++s) nrow[s] = (s < r) ? vals[s] : 0.f;
            } else {
#pragma unroll
                for (int s = 0; s < 64; ++s) vals[s] = (s <= r) ? -vals[s] : 0.f;
                tc::store_row64_bf16(sm + OFF_AQB, r, vals);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        if (*abort_s) break;

        // ================= P5: UT transform T = (I + A_kb)^{-1}
        ut_solve(NS, TS, PS, tid);
        if (tid < 64) {
            float vals[64];
            const float* trow = TS + tid * NSP;
#pragma unroll
            for (int s = 0; s < 64; ++s) vals[s] = (s <= tid) ? trow[s] : 0.f;
            tc::store_row64_bf16(sm + OFF_T, tid, vals);
        }
        tc::fence_async_smem();
        __syncthreads();

        // ================= P6: W^T = Kh^T T^T, Z^T = U^T A_kk^T
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id = tc::idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                tc::mma_bf16(tmem + TM_W, tc::desc_mnmajor(sbase + OFF_KH, 8192, kk),
                             tc::desc_kmajor(sbase + OFF_T, 8192, kk), id, kk > 0);
                tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_kmajor(sbase + OFF_L, 8192, kk), id, kk > 0);
            }
            tc::mma_commit(bar);
        }
        if (!tc::mbar_wait_bounded(bar, phase, WAIT_NS)) *abort_s = 1;
        phase ^= 1;
        tc::fence_after_sync();

        // ================= P7: W^T -> smem [i][r], Z^T -> smem [j][s]
        {
            float vals[64];
            const uint32_t col = grp == 0 ? TM_W : TM_Z;
            tc::tmem_ld32(tmem + lane_off + col, vals);
            tc::tmem_ld32(tmem + lane_off + col + 32, vals + 32);
            tc::tmem_wait_ld();
            tc::store_row64_bf16(sm + (grp == 0 ? OFF_W : OFF_ZT), gl, vals);
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();

        // ================= P8: E^T = S0^T W^T + Z^T T^T
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
            tc::mma_commit(bar);
        }
        if (!tc::mbar_wait_bounded(bar, phase, WAIT_NS)) *abort_s = 1;
        phase ^= 1;
        tc::fence_after_sync();

        // ================= P9: E^T -> smem [j][r]
        if (grp == 0) {
            float vals[64];
            tc::tmem_ld32(tmem + lane_off + TM_E, vals);
            tc::tmem_ld32(tmem + lane_off + TM_E + 32, vals + 32);
            tc::tmem_wait_ld();
            tc::store_row64_bf16(sm + OFF_ET, gl, vals);
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
                             tc::desc_kmajor(sbase + OFF_QH, 8192, kk), idKK, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_O, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_kmajor(sbase + OFF_AQK, 8192, kk), idMK, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_O, tc::desc_kmajor(sbase + OFF_ET, 16384, kk),
                             tc::desc_kmajor(sbase + OFF_AQB, 8192, kk), idKK, true);
            const uint32_t idMM = tc::idesc_bf16(128, 128, 1, 1);
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_U, 8192, kk),
                             tc::desc_mnmajor(sbase + OFF_KT, 8192, kk), idMM, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tmem + TM_S, tc::desc_kmajor(sbase + OFF_ET, 16384, kk),
                             tc::desc_mnmajor(sbase + OFF_BT, 8192, kk), idKM, true);
            tc::mma_commit(bar);
        }
        if (!tc::mbar_wait_bounded(bar, phase, WAIT_NS)) *abort_s = 1;
        phase ^= 1;
        tc::fence_after_sync();

        // ================= P11: outputs; bf16 copy of the new state
        if (grp == 0) {
            const int j = gl;
#pragma unroll 1
            for (int c0 = 0; c0 < 64; c0 += 32) {
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_O + c0, vals);
                tc::tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const int r = c0 + x;
                    if (r < n) o[(tok0 + r * row_stride) * D + j] = from_f32<Tin>(vals[x]);
                }
            }
        } else {
            const int j = gl;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
                tc::tmem_wait_ld();
                tc::store_row32_bf16(sm + OFF_S0T + (c0 >> 6) * 16384, j, (c0 >> 5) & 1, vals);
            }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        if (*abort_s) break;
    }

    if (*abort_s) {
        atomicOr(err_word, kErrTimeout);
        // let any product still in flight land before the memory is freed
        if (tid == 0) tc::mbar_wait_bounded(bar, phase, WAIT_NS);
        __syncthreads();
    } else if (s_final && grp == 1) {
        tc::fence_after_sync();
        const int j = gl;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_S + c0, vals);
            tc::tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) s_final[soff + (size_t)(c0 + x) * D + j] = vals[x];
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_free(tmem, 512);
    }
}

}  // namespace

bool chunked_tc_supports(const gdr_desc& d) {
    return d.in_dtype == GDR_BF16 && d.dk == D && d.dv == D && d.chunk == C;
}

cudaError_t launch_chunked_tc(const gdr_desc& d, const void* q, const void* k, const void* v,
                              const void* a, const void* b, const void* w, const float* s0,
                              void* o, float* s_final, int* err_word, cudaStream_t st) {
    using Tin = __nv_bfloat16;
    auto kern = chunked_tc_kernel<Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(d.B * d.H), NT, SMEM_BYTES, st>>>(
        d.B, d.T, d.H, (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)a,
        (const Tin*)b, (const Tin*)w, (int)d.decay, (int)d.erase, (int)d.write, s0, (Tin*)o,
        s_final, err_word);
    return cudaGetLastError();
}

}  // namespace gdr
