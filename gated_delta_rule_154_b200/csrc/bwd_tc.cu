// bwd_tc.cu -- gradients of the chunked gated delta rule on the Blackwell
// tensor cores (tcgen05, accumulators in tensor memory) fed by TMA: bf16
// inputs, dk = dv = 128, chunks of C = 64 tokens, one sequence per batch row.
//
// The pages train the recurrence through its chunkwise WY form (FG^2-GDN
// page, gist.science 2604.19021, section 2 "Methodology"); this file
// differentiates that form.  Per chunk (n <= 64 tokens, state S0 at its
// start, gamma_r = prod_{t<=r} a_t per key channel, mid token m = 31,
// g_m = gamma_m, gc = gamma_63 / g_m, Lam = gamma / g_m), with the operands
// of the forward kernel
//   Q' = Lam q, K' = Lam k, K" = k / Lam, B" = b K", U = w v, S~ = g_m S0
//   A_qk = tril(Q' K"^T), A_qb = tril(Q' B"^T)      (diagonal in)
//   A_kk = tril(K' K"^T), A_kb = tril(K' B"^T)      (strictly lower)
//   T = (I + A_kb)^-1,  E = T (K' S~ + A_kk U)       (the forward's key reads)
// and dS~ = gc dS_C (dS_C the gradient on the chunk's final state), the
// reverse of the chunk is
//   -dE = A_qb^T dO + B" dS~,       dU_p = A_qk^T dO + K" dS~
//   dY  = T^T dE,                   dU = dU_p + A_kk^T dY
//   D~  = dS~ + Q'^T dO + K'^T dY,  dS_0 = g_m D~      (dS_C of the chunk before)
//   dA  = [[dO (-E)^T, dO U^T], [dY (-E)^T, dY U^T]]  masked like the grams
//   XQ' = dO S~^T + dA_qb B" + dA_qk K",   XK' = dY S~^T + dA_kb B" + dA_kk K"
//   YB' = -E dS~^T + dA_qb^T Q' + dA_kb^T K',  YK' = U dS~^T + dA_qk^T Q' + dA_kk^T K'
// and the gradients follow elementwise:
//   dq = Lam XQ',  dk = Lam XK' + (YK' + b YB') / Lam,  db = K" YB'
//   dv = w dU,  dw = v dU,
//   dG = Q' XQ' + K' XK' - K" YK' - B" YB'  (+ rowsum(dS_C * S_C) at row n-1,
//        S_C the chunk's final state),  d log a_r = sum_{r' >= r} dG_r'.
// (The last term is the derivative of <dS_C, S_C> through gamma_63, which
// scales S_C as a whole.)  A float64 copy of these identities matched the
// oracle's backward to 1e-15 before this file was written.
//
// Three launches: the tcgen05 forward kernel in its state-writing
// instantiation (every chunk's S~ and E in bf16, exactly the tiles its own
// products read, and S_T in float32); bwd_tc_kernel, one CTA per (batch,
// head) walking the chunks from the last, which carries D~ in tensor memory
// and writes XQ', XK' (bf16, by TMA store), YK', YB', dU (bf16, from
// registers) and per chunk the G_C terms and gc; and bwd_epilogue_kernel, one warp per (batch, head,
// chunk), which forms the six gradients from them and the raw inputs (the
// reverse cumulative sum for da).  The G_C term of a chunk is rowsum(D~ S~)
// of the chunk after it (dS_C = g_m D~ and S_C = S~ / g_m there), and
// rowsum(dS_T S_T) for the last.
//
// Every product of bwd_tc_kernel is a 128-row tcgen05.mma with bf16 operands
// and float32 accumulation: 64-token operands are stacked in pairs ([Q'; K'],
// [B"; K"], [dO; dY], [-E; U]) so that one product yields two results, and
// where only one exists the other half of the A operand is a zero panel.
// The chain from dS~ to the next chunk's dS~ is three products (-dE, dY, D~)
// with a tensor-memory readout between them.
//
// Decay range as in the forward kernel: each channel's decay multiplied over
// tokens 1..31 and over 32..63 of a chunk must stay at or above 1e-35;
// otherwise GDR_ERR_RANGE.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "chunk_common.cuh"
#include "common.cuh"
#include "tc_common.cuh"

namespace gdr {

bool tc_map_bf16(CUtensorMap* m, const void* ptr, int B, int T, int H, int T_row);
bool tc_map_bf16_box32(CUtensorMap* m, const void* ptr, int B, int T, int H);
bool tc_map_state_bf16(CUtensorMap* m, const void* ptr, long long n_slots);
cudaError_t launch_chunked_tc_states(const gdr_desc& d, int T_row, const void* q, const void* k,
                                     const void* v, const void* a, const void* b,
                                     const void* w, const float* s0, float* s_final,
                                     void* s_tilde, int n_slots, int slot0, void* e_out,
                                     int* err_word, cudaStream_t st);

namespace {

constexpr int C = 64;         // chunk length
constexpr int D = 128;        // dk = dv
constexpr int NTC = 512;      // compute threads (warps 0-15)
constexpr int NT = NTC + 32;  // + the warp that issues every TMA copy and product

// ---- shared memory (bytes from a 1024-aligned base).  Operand tiles are
// 64-column panels of 128-byte swizzled rows (tc_common.cuh); a "128-row"
// tile has 16 KB panels, a "64-row" tile 8 KB panels.
constexpr uint32_t OFF_QK = 0;         // [Q'; K'] 128 rows (raw q lands in rows 0-63, k in 64-127)
constexpr uint32_t OFF_BK = 32768;     // [B"; K"] 128 rows (raw vector b / a in rows 0-63 / 64-127)
constexpr uint32_t OFF_DOY = 65536;    // [dO; dY] 128 rows (dO lands in rows 0-63)
constexpr uint32_t OFF_DS = 98304;     // S~ lands here [i][j] 128 rows, bf16; then dS~
constexpr uint32_t OFF_GQ = 131072;    // [A_qb | A_qk] 64 rows (r)
constexpr uint32_t OFF_TZA = 147456;   // T + I, zero, A_kk: three 64 x 64 panels, 8 KB each
constexpr uint32_t OFF_DE = 172032;    // dE 64 rows (raw vector w lands here)
constexpr uint32_t OFF_SCR = 188416;   // scratch, in turn:
constexpr uint32_t OFF_EIN = OFF_SCR;            //  loads: E 64 rows
constexpr uint32_t OFF_UIN = OFF_SCR + 16384;    //  loads: v 64 rows, replaced by U
constexpr uint32_t OFF_QT = OFF_SCR + 32768;     //  operand pass: float [8][128]
constexpr uint32_t OFF_NS = OFF_SCR;             //  solve: A_kb, float [64][68]
constexpr uint32_t OFF_TS = OFF_SCR + 17408;     //  solve: T, float [64][68]
constexpr uint32_t OFF_PS = OFF_SCR + 34816;     //  solve: float [2][16][16]
constexpr uint32_t OFF_DAT = OFF_SCR;            //  dA^T [s][r] 128 rows, bf16
constexpr uint32_t OFF_SMALL = OFF_SCR + 36864;
constexpr uint32_t OFF_GM = OFF_SMALL;           // float[128]: g_m of this chunk
constexpr uint32_t OFF_GC = OFF_SMALL + 512;     // float[128]: gc of this chunk
constexpr uint32_t OFF_GMN = OFF_SMALL + 1024;   // float[128]: g_m of the chunk after it
constexpr uint32_t OFF_SCA = OFF_SMALL + 1536;   // float[3][64]: scalar a, b, w
constexpr uint32_t OFF_EXP = OFF_SMALL + 2304;   // float[4][128]: partial G_C terms
constexpr uint32_t OFF_BAR = OFF_SMALL + 4352;
constexpr int NBAR = 12;
constexpr uint32_t OFF_TSLOT = OFF_BAR + 8 * NBAR;
constexpr uint32_t OFF_ABORT = OFF_TSLOT + 4;
constexpr uint32_t SMEM_USED = OFF_ABORT + 4;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(OFF_PS + 2048 <= OFF_SMALL && OFF_QT + 4096 <= OFF_SMALL, "scratch");

// ---- tensor-memory columns (512 allocated)
constexpr uint32_t TM_D = 0;     // D~ (lane = key channel i), float32, the running state gradient
constexpr uint32_t TM_G = 128;   // gram, then dA^T, then [YB'; YK']
constexpr uint32_t TM_Z = 256;   // [-dE -> dY; dU], then [XQ' | XK']^T
constexpr uint32_t TM_S = 384;   // S~ as a bf16 A operand (lane i, 64 columns)
constexpr uint32_t TM_EU = 448;  // [-E; U] as a bf16 A operand (lane s, 64 columns)

// The operand pass's tiles: Q', K' over raw q, k (QK); B", K" over raw b, a
// (BK); U over raw v; w in OFF_DE
__device__ __forceinline__ OpTiles op_tiles() {
    return OpTiles{OFF_QK, OFF_QK + 8192, OFF_BK + 8192, OFF_BK,     // q, k, a, b
                   OFF_QK, OFF_QK + 8192, OFF_BK + 8192, OFF_BK,     // Q', K', K", B"
                   OFF_UIN, OFF_DE};                                 // v -> U, w
}

constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr uint32_t BOX_BYTES = 64 * 128;     // one 64 x 64 bf16 TMA box

struct BwMaps {
    CUtensorMap q, k, v, a, b, w, dout, e;  // bf16 inputs (a/b/w only for vector gates)
    CUtensorMap sst;                        // the forward's S~ tiles
    CUtensorMap xq, xk;                     // bf16 intermediates, 32 x 32 boxes
    __nv_bfloat16 *yk, *yb, *du;            // bf16 intermediates written row by row
};

// XQ' and XK' (lane = channel in tensor memory) are transposed through 2 KB
// staging boxes of 32 tokens x 32 channels (64-byte rows, 64-byte swizzle:
// 16-byte chunk c of row r at c ^ ((r / 2) % 4)), each written and stored by
// TMA by one compute warp, in tiles that no load of the next chunk uses.
// YB', YK' and dU (lane = token) leave from registers, one 64-byte row piece
// per thread.
constexpr uint32_t SBOX = 2048;   // bytes of one staging box
// 32 values rounded to bf16, as four 16-byte stores to p (64-byte aligned)
__device__ __forceinline__ void st_row32_bf16(__nv_bfloat16* p, const float* v) {
    uint4* d = reinterpret_cast<uint4*>(p);
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
        uint4 u;
        u.x = tc::pack_bf16x2(v[8 * c16], v[8 * c16 + 1]);
        u.y = tc::pack_bf16x2(v[8 * c16 + 2], v[8 * c16 + 3]);
        u.z = tc::pack_bf16x2(v[8 * c16 + 4], v[8 * c16 + 5]);
        u.w = tc::pack_bf16x2(v[8 * c16 + 6], v[8 * c16 + 7]);
        d[c16] = u;
    }
}

// Barriers: TMA and tensor-core completions, then the compute threads'
// "ready" signals to the issuing warp (R_OP, R_GQ: thread 0 arrives after a
// compute barrier; R_DE, R_DY, R_DA: every compute warp arrives once its own
// lanes are done).  The compute warps issue the TMA loads and stores
// themselves.
enum : uint32_t {
    B_LD, B_G, B_Z1, B_Z3, B_A, B_XY, B_FIN,   // loads / gram / -dE / dY / D~,dU,dA / X,Y / all
    R_OP, R_GQ, R_DE, R_DY, R_DA                // ready for: gram / -dE / dY / D~,dU,dA / X,Y
};
static_assert(R_DA + 1 == NBAR, "barrier count");
__host__ __device__ constexpr uint32_t ready_count(uint32_t id) {
    return (id == R_DE || id == R_DY || id == R_DA) ? 16u : 1u;
}

// One row of 32 floats to global memory (16-byte stores).
__device__ __forceinline__ void store_row32_f32(float* dst, const float* v) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int x = 0; x < 8; ++x)
        d4[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
}

// The reverse sweep.  S~ of every chunk arrives through the sst map
// ([B*H][NC][128][128] bf16); sT [B*H][128][128] the final states; XQ', XK',
// YK', YB', dU leave through the bf16 maps; gce, gcs: [B*H][NC][128] the
// G_C terms and gc.
template <bool FG2>
__global__ void __launch_bounds__(NT, 1)
bwd_tc_kernel(const __grid_constant__ BwMaps maps, int B, int T, int H,
              const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
              const __nv_bfloat16* __restrict__ w, int a_kind, int b_kind, int w_kind,
              const float* __restrict__ ds_final, const float* __restrict__ sT, float* __restrict__ gce, float* __restrict__ gcs,
              float* __restrict__ ds0, int* __restrict__ err_word) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float* QT = reinterpret_cast<float*>(sm + OFF_QT);
    float* NS = reinterpret_cast<float*>(sm + OFF_NS);
    float* TS = reinterpret_cast<float*>(sm + OFF_TS);
    float* PS = reinterpret_cast<float*>(sm + OFF_PS);
    float* GM = reinterpret_cast<float*>(sm + OFF_GM);
    float* GC = reinterpret_cast<float*>(sm + OFF_GC);
    float* GMN = reinterpret_cast<float*>(sm + OFF_GMN);
    float* sca = reinterpret_cast<float*>(sm + OFF_SCA);
    float* EXP = reinterpret_cast<float*>(sm + OFF_EXP);
    volatile int* abort_s = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
    auto bar = [&](uint32_t id) { return sbase + OFF_BAR + 8u * id; };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quarter = warp & 3;                  // tensor-memory lanes 32*quarter ..
    const int cb = warp >> 2;                      // 32-column block this warp reads
    const int lane_t = 32 * quarter + (tid & 31);  // tensor-memory lane of this thread
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;

    const int bh = blockIdx.x;
    const int hi = bh % H, bi = bh / H;
    const int NC = (T + C - 1) / C;
    const size_t soff = (size_t)bh * D * D;
    const bool fb = b_kind == GDR_GATE_FG2, fw = w_kind == GDR_GATE_FG2;
    const bool va = a_kind == GDR_GATE_VECTOR, vb = b_kind == GDR_GATE_VECTOR || fb,
               vw = w_kind == GDR_GATE_VECTOR || fw;

    if (tid == 0) {
#pragma unroll 1
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(bar(i), ready_count(i));
        tc::mbar_fence_init();
        *abort_s = 0;
    }
    if (tid < D) GMN[tid] = 1.0f;
    // the zero panel of TZA, and the 16 x 16 blocks above the diagonal of
    // T + I (never written by the solve)
    if (tid < NTC) {
        const int r = tid >> 3, c16 = tid & 7;
        if ((c16 >> 1) > (r >> 4))
            *reinterpret_cast<uint4*>(sm + OFF_TZA + r * 128 + ((c16 ^ (r & 7)) << 4)) =
                make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + OFF_TZA + 8192 + 16 * tid) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (warp == 0) tc::tmem_alloc(sbase + OFF_TSLOT, 512);
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TSLOT);

    if (warp == NTC / 32) {
        // ======================= issuing warp (one thread)
        if ((tid & 31) == 0 && NC > 0) {
            tc::tma_prefetch_desc(&maps.q);
            tc::tma_prefetch_desc(&maps.k);
            tc::tma_prefetch_desc(&maps.v);
            tc::tma_prefetch_desc(&maps.dout);
            tc::tma_prefetch_desc(&maps.e);
            tc::tma_prefetch_desc(&maps.sst);
            uint32_t ph = 0;
            auto wait_ready = [&](uint32_t id, uint32_t parity) {
                if (!tc::mbar_wait_bounded(bar(id), parity, WAIT_NS)) { *abort_s = 1; return false; }
                tc::fence_after_sync();
                return *abort_s == 0;
            };
            const uint32_t idKK = tc::idesc_bf16(128, 128, 0, 0);
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t idMM = tc::idesc_bf16(128, 128, 1, 1);
#pragma unroll 1
            for (int c = NC - 1; c >= 0; --c, ph ^= 1) {
                // gram [Q'; K'] [B"; K"]^T; Z = [B"; K"] dS~; D~ += Q'^T dO
                if (!wait_ready(R_OP, ph)) break;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_G, tc::desc_kmajor(sbase + OFF_QK, 16384, kk),
                                 tc::desc_kmajor(sbase + OFF_BK, 16384, kk), idKK, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_Z, tc::desc_kmajor(sbase + OFF_BK, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_DS, 16384, kk), idKM, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_mnmajor(sbase + OFF_QK, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_DOY, 16384, kk), idMM, true);
                tc::mma_commit(bar(B_G));
                // Z += [A_qb^T; A_qk^T] dO: rows 0-63 become -dE, rows 64-127 dU_p
                if (!wait_ready(R_GQ, ph)) break;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_GQ, 8192, kk),
                                 tc::desc_mnmajor(sbase + OFF_DOY, 16384, kk), idMM, true);
                tc::mma_commit(bar(B_Z1));
                // Z += [T^T + I; 0] dE: rows 0-63 become dY
                if (!wait_ready(R_DE, ph)) break;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_TZA, 8192, kk),
                                 tc::desc_mnmajor(sbase + OFF_DE, 8192, kk), idMM, true);
                tc::mma_commit(bar(B_Z3));
                // D~ += K'^T dY;  Z += [0; A_kk^T] dY (rows 64-127 become dU);
                // dA^T = [-E; U] [dO; dY]^T
                if (!wait_ready(R_DY, ph)) break;
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_D, tc::desc_mnmajor(sbase + OFF_QK, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_DOY, 16384, kk), idMM, true);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_TZA + 8192, 8192, kk),
                                 tc::desc_mnmajor(sbase + OFF_DOY + 8192, 16384, kk), idMM, true);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16_ts(tmem + TM_G, tmem + TM_EU + 8 * kk,
                                    tc::desc_kmajor(sbase + OFF_DOY, 16384, kk), idKK, kk > 0);
                tc::mma_commit(bar(B_A));
                // [XQ' | XK']^T = S~ [dO; dY]^T + [B"; K"]^T dA^T   (lane = channel)
                // [YB'; YK']   = [-E; U] dS~^T + dA^T [Q'; K']      (lane = token)
                if (!wait_ready(R_DA, ph)) break;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16_ts(tmem + TM_Z, tmem + TM_S + 8 * kk,
                                    tc::desc_kmajor(sbase + OFF_DOY, 16384, kk), idKK, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_Z, tc::desc_mnmajor(sbase + OFF_BK, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_DAT, 16384, kk), idMM, true);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16_ts(tmem + TM_G, tmem + TM_EU + 8 * kk,
                                    tc::desc_kmajor(sbase + OFF_DS, 16384, kk), idKK, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_G, tc::desc_kmajor(sbase + OFF_DAT, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_QK, 16384, kk), idKM, true);
                tc::mma_commit(bar(B_XY));
            }
            // nothing of this CTA may still be in flight when it exits
            tc::mma_commit(bar(B_FIN));
            tc::mbar_wait_bounded(bar(B_FIN), 0, WAIT_NS);
        }
    } else {
        // ======================= compute warps
        // D~ = dS_T (unscaled: the first chunk's rescale takes it as dS_C)
        {
            float vals[32];
            if (ds_final) {
                const float4* src =
                    reinterpret_cast<const float4*>(ds_final + soff + (size_t)lane_t * D + 32 * cb);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float4 v4 = src[x];
                    vals[4 * x] = v4.x; vals[4 * x + 1] = v4.y;
                    vals[4 * x + 2] = v4.z; vals[4 * x + 3] = v4.w;
                }
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] = 0.f;
            }
            tc::tmem_st32(tmem + lane_off + TM_D + 32 * cb, vals);
            tc::tmem_wait_st();
        }
        // the G_C term of the last chunk: rowsum(dS_T * S_T), this thread's 32 columns
        if (NC > 0) {
            float part = 0.f;
            if (ds_final) {
                const float4* g4 = reinterpret_cast<const float4*>(ds_final + soff + (size_t)lane_t * D + 32 * cb);
                const float4* s4 = reinterpret_cast<const float4*>(sT + soff + (size_t)lane_t * D + 32 * cb);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float4 g = g4[x], sv = s4[x];
                    part = fmaf(g.x, sv.x, fmaf(g.y, sv.y, fmaf(g.z, sv.z, fmaf(g.w, sv.w, part))));
                }
            }
            EXP[cb * D + lane_t] = part;
        }
        // TMA loads of chunk cc's tiles: box j = 2 * tile + panel (q, k, do, E,
        // v, S~, b, a, w), spread over the compute warps.  B_LD is armed by
        // thread 0 before any box of the round can be issued.
        const uint32_t ld_bytes = (10u + (va ? 2u : 0u) + (vb ? 2u : 0u) + (vw ? 2u : 0u)) *
                                      BOX_BYTES + 2u * 16384u;
        auto issue_box = [&](int j, int cc) {
            const int t0l = cc * C;
            const uint32_t bl = bar(B_LD);
            const int p = j & 1, x = 64 * p;
            switch (j >> 1) {
            case 0: tc::tma_load_4d(sbase + OFF_QK + p * 16384, &maps.q, x, hi, t0l, bi, bl); break;
            case 1: tc::tma_load_4d(sbase + OFF_QK + p * 16384 + 8192, &maps.k, x, hi, t0l, bi, bl); break;
            case 2: tc::tma_load_4d(sbase + OFF_DOY + p * 16384, &maps.dout, x, hi, t0l, bi, bl); break;
            case 3: tc::tma_load_4d(sbase + OFF_EIN + p * 8192, &maps.e, x, hi, t0l, bi, bl); break;
            case 4: tc::tma_load_4d(sbase + OFF_UIN + p * 8192, &maps.v, x, hi, t0l, bi, bl); break;
            case 5: tc::tma_load_4d(sbase + OFF_DS + p * 16384, &maps.sst, x, 0, bh * NC + cc, 0, bl); break;
            case 6: if (vb) tc::tma_load_4d(sbase + OFF_BK + p * 16384, &maps.b, x, hi, t0l, bi, bl); break;
            case 7: if (va) tc::tma_load_4d(sbase + OFF_BK + p * 16384 + 8192, &maps.a, x, hi, t0l, bi, bl); break;
            default: if (vw) tc::tma_load_4d(sbase + OFF_DE + p * 8192, &maps.w, x, hi, t0l, bi, bl); break;
            }
        };
        // all 18 boxes, box j by warp j % 16
        auto issue_loads = [&](int cc) {
            if ((tid & 31) != 0) return;
#pragma unroll 1
            for (int j = warp; j < 18; j += 16) issue_box(j, cc);
        };
        int ld_out = 0;          // (thread 0) a load round issued and not yet waited for
        uint32_t ld_ph = 0;      // its phase parity
        if (NC > 0) {
            if (tid == 0) tc::mbar_arrive_expect_tx(bar(B_LD), ld_bytes);
            compute_sync();
            issue_loads(NC - 1);
            ld_out = 1;
        }
        // this warp's 32 x 32 box of a staged output out by TMA (rows past T
        // are not stored; a box starting past T is not issued)
        // element offset of token tok of this (batch, head) in a [B, T, H, 128] tensor
        auto row_off = [&](int tok) { return (((size_t)bi * T + tok) * H + hi) * D; };
        auto store_box = [&](const CUtensorMap* m, uint32_t box, int ch0, int tok0) {
            tc::fence_async_smem();
            __syncwarp();
            if ((tid & 31) == 0 && tok0 < T) {
                tc::tma_store_4d(m, sbase + box, ch0, hi, tok0, bi);
                tc::bulk_commit();
            }
        };
        uint32_t ph = 0;
        auto signal_or_stop = [&](uint32_t id) {
            const bool stop = compute_sync_or(*abort_s != 0);
            if (tid == 0) tc::mbar_arrive(bar(id));
            return stop;
        };
        // each warp signals `id` once its own lanes are done (no CTA barrier)
        auto warp_signal = [&](uint32_t id) {
            __syncwarp();
            if ((tid & 31) == 0) tc::mbar_arrive(bar(id));
        };
        // every thread waits on a product's commit itself; a wait that runs out
        // sets the abort flag (the vote at the chunk's end stops all threads)
        auto wait_each = [&](uint32_t id, uint32_t parity) {
            if (!*abort_s && !tc::mbar_wait_bounded(bar(id), parity, WAIT_NS)) *abort_s = 1;
            tc::fence_after_sync();
        };
#pragma unroll 1
        for (int c = NC - 1; c >= 0; --c, ph ^= 1) {
            const int t0 = c * C;
            const int n = min(C, T - t0);
            // ================= C1: scalar gates, the chunk's tiles, the operand pass
            if (tid < C) {
                const long long tok = ((long long)bi * T + t0 + tid) * H + hi;
                const bool in = tid < n;
                sca[tid] = (a_kind == GDR_GATE_SCALAR && in) ? to_f32(a[tok]) : 1.f;
                sca[64 + tid] = (b_kind == GDR_GATE_SCALAR && in) ? to_f32(b[tok]) : 1.f;
                sca[128 + tid] = (w_kind == GDR_GATE_SCALAR && in) ? to_f32(w[tok]) : 1.f;
            }
            if (tid == 0) {
                if (!*abort_s && !tc::mbar_wait_bounded(bar(B_LD), ph, WAIT_NS)) *abort_s = 1;
                else ld_out = 0;
            }
            if (compute_sync_or(*abort_s != 0)) break;
            operand_pass<false, FG2>(sm, op_tiles(), tid, va, vb, vw, fb, fw, a_kind, n, sca, QT,
                                     err_word, [] {},
                                     [&](int i, float g_m, float g_c) {
                                         GM[i] = g_m;
                                         GC[i] = g_c;
                                     });
            compute_sync();
            // ================= C1b: [-E; U] and S~ into tensor memory; the rescale
            {
                // [-E; U]: lane s of the stack, 32 value columns
                const int s = lane_t & 63;
                const uint8_t* src = sm + (lane_t < 64 ? OFF_EIN : OFF_UIN) + (cb >> 1) * 8192 + s * 128;
                const uint32_t flip = lane_t < 64 ? 0x80008000u : 0u;
                uint32_t words[16];
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int c16 = 4 * (cb & 1) + qd;
                    const uint4 u = *reinterpret_cast<const uint4*>(src + ((c16 ^ (s & 7)) << 4));
                    words[4 * qd] = u.x ^ flip;
                    words[4 * qd + 1] = u.y ^ flip;
                    words[4 * qd + 2] = u.z ^ flip;
                    words[4 * qd + 3] = u.w ^ flip;
                }
                tc::tmem_st16(tmem + lane_off + TM_EU + 16 * cb, words);
            }
            {
                // S~ (the forward's tile, landed in OFF_DS) -> tensor memory: lane i,
                // 32 value columns; this thread later overwrites exactly these bytes
                // with dS~
                const uint8_t* src = sm + OFF_DS + (cb >> 1) * 16384 + lane_t * 128;
                uint32_t words[16];
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int c16 = 4 * (cb & 1) + qd;
                    const uint4 u = *reinterpret_cast<const uint4*>(src + ((c16 ^ (lane_t & 7)) << 4));
                    words[4 * qd] = u.x;
                    words[4 * qd + 1] = u.y;
                    words[4 * qd + 2] = u.z;
                    words[4 * qd + 3] = u.w;
                }
                tc::tmem_st16(tmem + lane_off + TM_S + 16 * cb, words);
            }
            {
                // dS_C = g_m(next) D~;  dS~ = gc dS_C into tensor memory and, bf16,
                // into OFF_DS
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_D + 32 * cb, vals);
                tc::tmem_wait_ld();
                const float f = GMN[lane_t] * GC[lane_t];
#pragma unroll
                for (int x = 0; x < 32; ++x) vals[x] *= f;
                tc::tmem_st32(tmem + lane_off + TM_D + 32 * cb, vals);
                tc::store_row32_bf16(sm + OFF_DS + (cb >> 1) * 16384, lane_t, cb & 1, vals);
            }
            tc::tmem_wait_st();
            tc::fence_async_smem();
            // the last chunk's XQ' / XK' stores have read their boxes (the dY
            // rows and the [A_qb | A_qk] tile are rewritten after this barrier)
            if ((tid & 31) == 0) tc::bulk_wait_read();
            __syncwarp();
            tc::fence_before_sync();
            if (signal_or_stop(R_OP)) break;

            // ================= C2: the G_C term out; the gram's blocks
            if (tid < D) {
                gce[((size_t)bh * NC + c) * D + tid] =
                    (EXP[tid] + EXP[D + tid]) + (EXP[2 * D + tid] + EXP[3 * D + tid]);
                gcs[((size_t)bh * NC + c) * D + tid] = GC[tid];
                GMN[tid] = GM[tid];
            }
            wait_each(B_G, ph);
            {
                // rows r of Q' (lanes 0-63) or K' (lanes 64-127); this warp's 32 x 32
                // block lies below (mode < 0), on (0) or above (> 0) the diagonal
                // of its 64 x 64 gram block: warp-uniform
                const bool top = lane_t < 64;
                const int r = lane_t & 63;
                const int s0c = 32 * (cb & 1);
                const int mode = (cb & 1) - (quarter & 1);
                float vals[32];
                if (mode > 0) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) vals[x] = 0.f;
                } else {
                    tc::tmem_ld32(tmem + lane_off + TM_G + 32 * cb, vals);
                    tc::tmem_wait_ld();
                    if (mode == 0) {
                        const int lim = top ? r - s0c + 1 : r - s0c;
#pragma unroll
                        for (int x = 0; x < 32; ++x) vals[x] = x < lim ? vals[x] : 0.f;
                    }
                }
                if (top) {           // A_qb (cb 0-1), A_qk (cb 2-3)
                    tc::store_row32_bf16(sm + OFF_GQ + (cb >> 1) * 8192, r, cb & 1, vals);
                } else if (cb < 2) { // A_kb, for the solve
                    float* nrow = NS + r * NSP + s0c;
#pragma unroll
                    for (int x = 0; x < 32; x += 4)
                        st4(nrow + x, make_float4(vals[x], vals[x + 1], vals[x + 2], vals[x + 3]));
                } else {             // A_kk
                    tc::store_row32_bf16(sm + OFF_TZA + 16384, r, cb & 1, vals);
                }
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            if (signal_or_stop(R_GQ)) break;

            // ================= C3: warps 8-15 solve T + I; warps 0-7 read -dE
            if (warp >= 8) {
                ut_solve<2>(NS, TS, PS, sm + OFF_TZA, tid - 256);
                tc::fence_async_smem();
            } else {
                wait_each(B_Z1, ph);
                if (quarter < 2) {  // warps 0, 1, 4, 5: lanes 0-63, 64 columns each
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float vals[32];
                        tc::tmem_ld32(tmem + lane_off + TM_Z + 64 * cb + 32 * hh, vals);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) vals[x] = -vals[x];
                        tc::store_row32_bf16(sm + OFF_DE + cb * 8192, lane_t, hh, vals);
                    }
                }
                tc::fence_async_smem();
            }
            tc::fence_before_sync();
            warp_signal(R_DE);

            // ================= C4: dY -> rows 64-127 of [dO; dY]
            wait_each(B_Z3, ph);
            if (quarter < 2) {
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_Z + 32 * cb, vals);
                tc::tmem_wait_ld();
                tc::store_row32_bf16(sm + OFF_DOY + (cb >> 1) * 16384, 64 + lane_t, cb & 1, vals);
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            warp_signal(R_DY);

            // ================= C5: dA^T masked -> bf16; dU out
            wait_each(B_A, ph);
            // arm B_LD for the next chunk's boxes: they are issued only after the
            // X / Y products, which wait for every warp's R_DA below
            if (tid == 0 && c > 0) {
                tc::mbar_arrive_expect_tx(bar(B_LD), ld_bytes);
                ld_out = 1;
                ld_ph = ph ^ 1;
            }
            if (c > 0) {
                // the G_C term of the chunk before: rowsum(dS_C * S_C) with dS_C =
                // g_m D~ and S_C = S~ / g_m (this chunk's start), i.e. rowsum(D~ * S~)
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_D + 32 * cb, vals);
                uint32_t sw[16];
                tc::tmem_ld16u(tmem + lane_off + TM_S + 16 * cb, sw);
                tc::tmem_wait_ld();
                float part = 0.f;
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    part = fmaf(vals[2 * x], __uint_as_float(sw[x] << 16), part);
                    part = fmaf(vals[2 * x + 1], __uint_as_float(sw[x] & 0xFFFF0000u), part);
                }
                EXP[cb * D + lane_t] = part;
            }
            {
                // lane s of [-E; U], columns r of [dO; dY]: keep r >= s against dO,
                // r > s against dY; block relation as for the gram
                const int s = lane_t & 63;
                const int rb = 32 * (cb & 1);
                const int mode = (quarter & 1) - (cb & 1);
                float vals[32];
                if (mode > 0) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) vals[x] = 0.f;
                } else {
                    tc::tmem_ld32(tmem + lane_off + TM_G + 32 * cb, vals);
                    tc::tmem_wait_ld();
                    if (mode == 0) {
                        const int lim = s - rb + (cb >= 2 ? 1 : 0);  // keep x >= lim
#pragma unroll
                        for (int x = 0; x < 32; ++x) vals[x] = x >= lim ? vals[x] : 0.f;
                    }
                }
                tc::store_row32_bf16(sm + OFF_DAT + (cb >> 1) * 16384, lane_t, cb & 1, vals);
            }
            if (quarter >= 2) {   // dU: token lane_t - 64, this warp's 32 channels
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_Z + 32 * cb, vals);
                tc::tmem_wait_ld();
                const int tok = t0 + (lane_t & 63);
                if (tok < T) st_row32_bf16(maps.du + row_off(tok) + 32 * cb, vals);
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            warp_signal(R_DA);

            // ================= C6: [YB'; YK'] and [XQ' | XK']^T out
            wait_each(B_XY, ph);
            // the next chunk's tiles: nothing below stages into their tiles
            if (c > 0) issue_loads(c - 1);
            {
                // [YB'; YK']: lane = token, this warp's 32 channels 32cb..
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_G + 32 * cb, vals);
                tc::tmem_wait_ld();
                const int tok = t0 + (lane_t & 63);
                if (tok < T) st_row32_bf16((quarter < 2 ? maps.yb : maps.yk) + row_off(tok) + 32 * cb, vals);
            }
            {
                // [XQ' | XK']^T: lane = channel, columns = tokens; this warp's
                // channels 32q.. and tokens 32(cb & 1).. into a [token][channel]
                // box, staged where no load lands: the dY rows of [dO; dY]
                // (XQ') and the [A_qb | A_qk] tile (XK')
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_Z + 32 * cb, vals);
                tc::tmem_wait_ld();
                const int bx = 2 * quarter + (cb & 1);
                const uint32_t box = cb < 2 ? OFF_DOY + (bx >> 2) * 16384 + 8192 + (bx & 3) * SBOX
                                            : OFF_GQ + bx * SBOX;
                const int cl = tid & 31;
                uint8_t* dst = sm + box + 2 * (cl & 7);
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    *reinterpret_cast<__nv_bfloat16*>(dst + 64 * x +
                                                      (((cl >> 3) ^ ((x >> 1) & 3)) << 4)) =
                        __float2bfloat16_rn(vals[x]);
                store_box(cb < 2 ? &maps.xq : &maps.xk, box, 32 * quarter, t0 + 32 * (cb & 1));
            }
            // (the X^T stores are waited for before the next chunk's R_OP)
            tc::fence_before_sync();
            if (compute_sync_or(*abort_s != 0)) break;
        }
        // nothing this CTA started may still be in flight when it exits
        if (tid == 0 && ld_out) tc::mbar_wait_bounded(bar(B_LD), ld_ph, WAIT_NS);
        if ((tid & 31) == 0) tc::bulk_wait_all();
        // dS0 = g_m(first chunk) D~
        if (ds0 && NC > 0 && !compute_sync_or(*abort_s != 0)) {
            float vals[32];
            tc::tmem_ld32(tmem + lane_off + TM_D + 32 * cb, vals);
            tc::tmem_wait_ld();
            const float g = GMN[lane_t];
#pragma unroll
            for (int x = 0; x < 32; ++x) vals[x] *= g;
            store_row32_f32(ds0 + soff + (size_t)lane_t * D + 32 * cb, vals);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (*abort_s) {
        if (tid == 0) atomicOr(err_word, kErrTimeout);
    }
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_free(tmem, 512);
    }
}

// ---------------------------------------------------------------- epilogue
// One warp per (batch, head, chunk), lane l = channels 4l .. 4l+3, the
// chunk's tokens from the last: from the raw inputs and the reverse sweep's
// XQ', XK', YK', YB', dU, G_C terms and gc,
//   Lam_63 = gc, Lam_{r-1} = Lam_r / a_r   (= gamma_{r-1} / g_m)
//   dq = Lam XQ', dk = Lam XK' + (YK' + b YB') / Lam, db = K" YB',
//   dv = w dU, dw = v dU, d log a_r = sum_{r' >= r} dG_r', da = d log a / a.
// Scalar gates take the sum over channels (a warp reduction).  FG^2-GDN
// learning rates: the gradients of the key sqrt(beta^k) k and write gate
// sqrt(beta^v) carried through the square roots (dk = sqrt(beta^k) dk~,
// dbeta^k = k dk~ / (2 sqrt(beta^k)), dbeta^v = v dU / (2 sqrt(beta^v))).
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}
__device__ __forceinline__ void st_bf16x4(__nv_bfloat16* p, const float* f) {
    *reinterpret_cast<uint2*>(p) =
        make_uint2(tc::pack_bf16x2(f[0], f[1]), tc::pack_bf16x2(f[2], f[3]));
}
__device__ __forceinline__ void ld_f32x4(const float* p, float* f) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
__global__ void __launch_bounds__(128)
bwd_epilogue_kernel(int T, int H, int NC, long long n_units, const __nv_bfloat16* __restrict__ q,
                    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                    const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                    const __nv_bfloat16* __restrict__ w, int a_kind, int b_kind, int w_kind,
                    const __nv_bfloat16* __restrict__ xq, const __nv_bfloat16* __restrict__ xk,
                    const __nv_bfloat16* __restrict__ yk, const __nv_bfloat16* __restrict__ yb,
                    const __nv_bfloat16* __restrict__ du, const float* __restrict__ gce,
                    const float* __restrict__ gcs, __nv_bfloat16* __restrict__ dq,
                    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                    __nv_bfloat16* __restrict__ da, __nv_bfloat16* __restrict__ db,
                    __nv_bfloat16* __restrict__ dw) {
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (unit >= n_units) return;
    const int c = (int)(unit % NC);
    const long long bh = unit / NC;
    const int hi = (int)(bh % H), bi = (int)(bh / H);
    const int t0 = c * C, n = min(C, T - t0);
    const int i0 = 4 * lane;
    const bool fb = b_kind == GDR_GATE_FG2, fw = w_kind == GDR_GATE_FG2;
    const long long tok0 = ((long long)bi * T + t0) * H + hi;   // token-head index of row 0
    float lam[4], cum[4] = {0.f, 0.f, 0.f, 0.f}, gterm[4];
    ld_f32x4(gcs + (bh * NC + c) * D + i0, lam);
    ld_f32x4(gce + (bh * NC + c) * D + i0, gterm);
    // one token's inputs, still packed (bf16 x 4 per tensor); the next
    // token's are loaded while this one is processed
    struct Tok {
        uint2 q, k, v, a, b, w, xq, xk, yk, yb, du;
    };
    auto gate4 = [&](const __nv_bfloat16* g, int kind, long long th, long long tv) -> uint2 {
        if (kind == GDR_GATE_ONE) return make_uint2(0x3F803F80u, 0x3F803F80u);
        if (kind == GDR_GATE_SCALAR) {
            const uint32_t s1 = *reinterpret_cast<const uint16_t*>(g + th);
            return make_uint2(s1 | (s1 << 16), s1 | (s1 << 16));
        }
        return *reinterpret_cast<const uint2*>(g + tv);
    };
    auto load_tok = [&](int r, Tok& t) {
        const long long th = tok0 + (long long)r * H, tv = th * D + i0;
        t.q = *reinterpret_cast<const uint2*>(q + tv);
        t.k = *reinterpret_cast<const uint2*>(k + tv);
        t.v = *reinterpret_cast<const uint2*>(v + tv);
        t.a = gate4(a, a_kind, th, tv);
        t.b = gate4(b, b_kind, th, tv);
        t.w = gate4(w, w_kind, th, tv);
        t.xq = *reinterpret_cast<const uint2*>(xq + tv);
        t.xk = *reinterpret_cast<const uint2*>(xk + tv);
        t.yk = *reinterpret_cast<const uint2*>(yk + tv);
        t.yb = *reinterpret_cast<const uint2*>(yb + tv);
        t.du = *reinterpret_cast<const uint2*>(du + tv);
    };
    auto unpack = [](uint2 u, float* f) {
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xFFFF0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xFFFF0000u);
    };
    Tok cur, nxt;
    if (n > 0) load_tok(n - 1, cur);
#pragma unroll 1
    for (int r = n - 1; r >= 0; --r) {
        if (r > 0) load_tok(r - 1, nxt);
        const long long th = tok0 + (long long)r * H, tv = th * D + i0;
        float qv[4], kv[4], vv[4], av[4], bv[4], wv[4], XQ[4], XK[4], YK[4], YB[4], dU[4];
        unpack(cur.q, qv);
        unpack(cur.k, kv);
        unpack(cur.v, vv);
        unpack(cur.a, av);
        unpack(cur.b, bv);
        unpack(cur.w, wv);
        unpack(cur.xq, XQ);
        unpack(cur.xk, XK);
        unpack(cur.yk, YK);
        unpack(cur.yb, YB);
        unpack(cur.du, dU);
        float oq[4], ok[4], ov[4], oa[4], ob[4], ow[4];
        float sb = 0.f, sw = 0.f, sa = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float lm = lam[x], li = 1.f / lm;
            const float sbk = fb ? sqrt_fast(fmaxf(bv[x], 0.f)) : 1.f;   // sqrt(beta^k)
            const float kt = kv[x] * sbk;                                 // the key used
            const float bt = fb ? 1.f : bv[x];                            // the erase gate used
            const float wt = fw ? sqrt_fast(fmaxf(wv[x], 0.f)) : wv[x];   // the write gate used
            const float Kpp = li * kt;
            float dG = lm * (qv[x] * XQ[x] + kt * XK[x]) - Kpp * (YK[x] + bt * YB[x]);
            if (r == n - 1) dG += gterm[x];
            cum[x] += dG;
            const float dkt = lm * XK[x] + li * (YK[x] + bt * YB[x]);
            oq[x] = lm * XQ[x];
            ok[x] = dkt * sbk;
            ov[x] = wt * dU[x];
            ob[x] = fb ? kv[x] * dkt / (2.f * sbk) : Kpp * YB[x];
            ow[x] = fw ? vv[x] * dU[x] / (2.f * wt) : vv[x] * dU[x];
            oa[x] = cum[x] / av[x];
            sb += ob[x];
            sw += ow[x];
            sa += cum[x];
        }
        st_bf16x4(dq + tv, oq);
        st_bf16x4(dk + tv, ok);
        st_bf16x4(dv + tv, ov);
        if (a_kind == GDR_GATE_VECTOR) st_bf16x4(da + tv, oa);
        if (b_kind == GDR_GATE_VECTOR || fb) st_bf16x4(db + tv, ob);
        if (w_kind == GDR_GATE_VECTOR || fw) st_bf16x4(dw + tv, ow);
        if (a_kind == GDR_GATE_SCALAR) {
            sa = warp_sum(sa);
            if (lane == 0) da[th] = __float2bfloat16_rn(sa / av[0]);
        }
        if (b_kind == GDR_GATE_SCALAR) {
            sb = warp_sum(sb);
            if (lane == 0) db[th] = __float2bfloat16_rn(sb);
        }
        if (w_kind == GDR_GATE_SCALAR) {
            sw = warp_sum(sw);
            if (lane == 0) dw[th] = __float2bfloat16_rn(sw);
        }
        // Lam of the token before
#pragma unroll
        for (int x = 0; x < 4; ++x) lam[x] /= av[x];
        cur = nxt;
    }
}

inline size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

struct TcWorkspace {
    void* states;    // [B*H][NC][128][128] bf16 S~
    float* sT;       // [B*H][128][128]
    void* e;         // [B, T, H, 128] bf16
    void* pre[5];    // XQ', XK', YK', YB', dU: [B, T, H, 128] bf16
    float* gce;      // [B*H][NC][128] G_C terms
    float* gcs;      // [B*H][NC][128] gc per chunk and channel
    size_t bytes;
};

TcWorkspace carve(const gdr_desc& d, void* base) {
    const size_t bh = (size_t)d.B * d.H, nc = ((size_t)d.T + C - 1) / C;
    const size_t tok = (size_t)d.B * d.T * d.H;
    TcWorkspace w;
    uint8_t* p = static_cast<uint8_t*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* r = p ? p + off : nullptr;
        off += round256(bytes);
        return r;
    };
    w.states = take(bh * nc * D * D * 2);
    w.sT = reinterpret_cast<float*>(take(bh * D * D * 4));
    w.e = take(tok * D * 2);
    for (int x = 0; x < 5; ++x) w.pre[x] = take(tok * D * 2);
    w.gce = reinterpret_cast<float*>(take(bh * nc * D * 4));
    w.gcs = reinterpret_cast<float*>(take(bh * nc * D * 4));
    w.bytes = off;
    return w;
}

}  // namespace

// The tensor-core backward handles bf16, dk = dv = 128, one sequence per
// batch row, at least one token.
bool backward_tc_supports(const gdr_desc& d, bool packed) {
    return !packed && d.in_dtype == GDR_BF16 && d.dk == D && d.dv == D && d.T > 0;
}

size_t backward_tc_workspace_bytes(const gdr_desc& d) { return carve(d, nullptr).bytes; }

// in = {q, k, v, a, b, w}; grads = {dq, dk, dv, da, db, dw}.
cudaError_t launch_backward_tc(const gdr_desc& d, const void* const* in, const float* s0,
                               const void* dout, const float* ds_final, void* const* grads,
                               float* ds0, void* workspace, int* err_word, cudaStream_t st) {
    const TcWorkspace ws = carve(d, workspace);
    const int NC = (d.T + C - 1) / C;
    gdr_desc f = d;
    f.chunk = C;
    cudaError_t e = launch_chunked_tc_states(f, d.T, in[0], in[1], in[2], in[3], in[4], in[5], s0,
                                             ws.sT, ws.states, NC, 0, ws.e, err_word, st);
    if (e != cudaSuccess) return e;

    BwMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int B = d.B, T = d.T, H = d.H;
    bool ok = tc_map_bf16(&maps.q, in[0], B, T, H, T) && tc_map_bf16(&maps.k, in[1], B, T, H, T) &&
              tc_map_bf16(&maps.v, in[2], B, T, H, T) &&
              tc_map_bf16(&maps.dout, dout, B, T, H, T) && tc_map_bf16(&maps.e, ws.e, B, T, H, T);
    if (ok && d.decay == GDR_GATE_VECTOR) ok = tc_map_bf16(&maps.a, in[3], B, T, H, T);
    if (ok && (d.erase == GDR_GATE_VECTOR || d.erase == GDR_GATE_FG2))
        ok = tc_map_bf16(&maps.b, in[4], B, T, H, T);
    if (ok && (d.write == GDR_GATE_VECTOR || d.write == GDR_GATE_FG2))
        ok = tc_map_bf16(&maps.w, in[5], B, T, H, T);
    ok = ok && tc_map_bf16_box32(&maps.xq, ws.pre[0], B, T, H) &&
         tc_map_bf16_box32(&maps.xk, ws.pre[1], B, T, H) &&
         tc_map_state_bf16(&maps.sst, ws.states, (long long)B * H * NC);
    maps.yk = static_cast<__nv_bfloat16*>(ws.pre[2]);
    maps.yb = static_cast<__nv_bfloat16*>(ws.pre[3]);
    maps.du = static_cast<__nv_bfloat16*>(ws.pre[4]);
    if (!ok) return cudaErrorInvalidValue;

    const bool fg2 = d.erase == GDR_GATE_FG2 || d.write == GDR_GATE_FG2;
    auto kern = fg2 ? bwd_tc_kernel<true> : bwd_tc_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const auto* a = static_cast<const __nv_bfloat16*>(in[3]);
    const auto* b = static_cast<const __nv_bfloat16*>(in[4]);
    const auto* w = static_cast<const __nv_bfloat16*>(in[5]);
    kern<<<(unsigned)((long long)B * H), NT, SMEM_BYTES, st>>>(
        maps, B, T, H, a, b, w, (int)d.decay, (int)d.erase, (int)d.write, ds_final, ws.sT,
        ws.gce, ws.gcs, ds0, err_word);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const long long units = (long long)B * H * NC;
    bwd_epilogue_kernel<<<(unsigned)((units + 3) / 4), 128, 0, st>>>(
        T, H, NC, units, static_cast<const __nv_bfloat16*>(in[0]),
        static_cast<const __nv_bfloat16*>(in[1]), static_cast<const __nv_bfloat16*>(in[2]), a, b,
        w, (int)d.decay, (int)d.erase, (int)d.write,
        static_cast<const __nv_bfloat16*>(ws.pre[0]), static_cast<const __nv_bfloat16*>(ws.pre[1]),
        static_cast<const __nv_bfloat16*>(ws.pre[2]), static_cast<const __nv_bfloat16*>(ws.pre[3]),
        static_cast<const __nv_bfloat16*>(ws.pre[4]), ws.gce, ws.gcs, static_cast<__nv_bfloat16*>(grads[0]),
        static_cast<__nv_bfloat16*>(grads[1]), static_cast<__nv_bfloat16*>(grads[2]),
        static_cast<__nv_bfloat16*>(grads[3]), static_cast<__nv_bfloat16*>(grads[4]),
        static_cast<__nv_bfloat16*>(grads[5]));
    return cudaGetLastError();
}

}  // namespace gdr
