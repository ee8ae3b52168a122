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
// One CTA (16 compute warps and one issuing warp) owns one (batch, head)
// and walks its chunks in order; S~ stays in float32 in tensor memory (lane =
// key channel) for the whole sequence.  Raw q/k/v and vector gates arrive by
// TMA as 64-token x 64-channel boxes, 128-byte swizzled, i.e. already in the
// operand layout of tc_common.cuh, each prefetched as soon as its
// destination is free; o leaves by a TMA store.  Products are tcgen05.mma
// issued by one thread of the issuing warp; the decay products, the UT solve
// and the conversions run on the CUDA cores with 8- and 16-byte
// shared-memory accesses.  The compute threads wait on the TMA and product
// barriers themselves and tell the issuing warp per warp that an operand set
// is in place; a CTA barrier stands only where data crosses warps, and one
// vote per chunk stops all threads together after a wait ran out.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "chunk_common.cuh"
#include "common.cuh"
#include "tc_common.cuh"

namespace gdr {
namespace {

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // dk = dv
constexpr int NTC = 512;     // compute threads (warps 0-15)
constexpr int NT = NTC + 32; // + one warp that issues every TMA copy and tensor-core product

// ---- shared memory map (bytes from a 1024-aligned base).  Operand tiles are
// 64-column panels of 128-byte swizzled rows; "rows r" below are tokens.
constexpr uint32_t OFF_RAW = 0;         // raw k (rows 0-63) and q (rows 64-127), 2 panels
constexpr uint32_t OFF_X1 = 32768;      // raw vector a and b land here (rows 0-63 / 64-127),
                                        // replaced in place by [K'; Q'] 128 x 128
constexpr uint32_t OFF_X2 = 65536;      // [K"; B"] 128 x 128; between the state products
                                        // and P6 the K" rows hold R (bf16)
constexpr uint32_t OFF_U = 98304;       // U = w*v [s][j] 64 x 128 (raw v lands here)
constexpr uint32_t OFF_W = 114688;      // raw vector w 64 x 128
constexpr uint32_t OFF_Z3 = 131072;     // [T - I; 0; -A_qb] 192 x 64
constexpr uint32_t OFF_S0 = 155648;     // S~ [i][j] bf16 128 x 128
constexpr uint32_t OFF_R = 188416;      // scratch region:
constexpr uint32_t OFF_NS = OFF_R;              //  P4-P5: A_kb, float [64][68]
constexpr uint32_t OFF_TS = OFF_R + 17408;      //  P5: T, float [64][68]
constexpr uint32_t OFF_PS = OFF_R + 34816;      //  P5: float [2][16][16]
constexpr uint32_t OFF_EB = OFF_R;              //  P7 -> next P1: E bf16 [s][j] 64 x 128
constexpr uint32_t OFF_OST = OFF_R + 16384;     //  next P1 -> o store: staging [r][j] 64 x 128
constexpr uint32_t OFF_QT = OFF_R + 32768;      //  P1: float [8][128], 8-token products
                                                //  (clear of EB, which the previous chunk's
                                                //  state update still reads, and of OST)
constexpr uint32_t OFF_SMALL = OFF_R + 37888;   // 226304
constexpr uint32_t OFF_FCUR = OFF_SMALL;        // float[128]: state scale this chunk
constexpr uint32_t OFF_FPREV = OFF_SMALL + 512; // float[128]: gamma_C/g_m of last chunk
constexpr uint32_t OFF_SCA = OFF_SMALL + 1024;  // float[2][3][64]: scalar a, b, w (2 chunks)
constexpr uint32_t OFF_BAR = OFF_SMALL + 3072;  // NBAR mbarriers (see the kernel)
constexpr int NBAR = 14;
constexpr uint32_t OFF_TSLOT = OFF_BAR + 8 * NBAR;
constexpr uint32_t OFF_ABORT = OFF_TSLOT + 4;
constexpr uint32_t SMEM_USED = OFF_ABORT + 4;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(OFF_PS + 2 * 256 * 4 <= OFF_SMALL, "solve scratch");
static_assert(OFF_QT >= OFF_OST + 16384 && OFF_QT + 8 * 128 * 4 <= OFF_SMALL, "QT placement");

// ---- tensor-memory columns (512 allocated)
constexpr uint32_t TM_G = 0;     // gram 128 x 128
constexpr uint32_t TM_X = 128;   // [R -> E; O] 128 x 128
constexpr uint32_t TM_S = 256;   // S~ 128 x 128 (lane = key channel), float32 state
constexpr uint32_t TM_AQ = 384;  // A operand [A_kk; A_qk] 128 x 64 bf16 (32 columns)

__device__ __forceinline__ OpTiles op_tiles() {
    return OpTiles{OFF_RAW + 8192, OFF_RAW, OFF_X1, OFF_X1 + 8192,   // q, k, a, b
                   OFF_X1 + 8192, OFF_X1, OFF_X2, OFF_X2 + 8192,     // Q', K', K", B"
                   OFF_U, OFF_W};                                     // v -> U, w
}

constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr uint32_t BOX_BYTES = 64 * 128;     // one 64 x 64 bf16 TMA box
constexpr uint32_t IDESC_NEG_B = 1u << 14;   // negate the B operand

struct TcMaps {
    CUtensorMap q, k, v, a, b, w, o;  // a/b/w only meaningful for vector gates
    CUtensorMap sst;                  // state-writing instantiation: S~ tiles
};

// ---------------------------------------------------------------- TMA issue
// Group "kqw": raw k and q into RAW, vector w into W.  Group "ab": vector a
// and b into X1.  Group "v": v into U.
__device__ __forceinline__ void issue_kqw(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                          bool vw, uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 2u * (2u + (vw ? 1u : 0u)) * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384, &m.k, 64 * p, hi, t0, bi, bar);
        tc::tma_load_4d(sbase + OFF_RAW + p * 16384 + 8192, &m.q, 64 * p, hi, t0, bi, bar);
        if (vw) tc::tma_load_4d(sbase + OFF_W + p * 8192, &m.w, 64 * p, hi, t0, bi, bar);
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

__device__ __forceinline__ void issue_v(const TcMaps& m, uint32_t sbase, int t0, int hi, int bi,
                                        uint32_t bar) {
    tc::mbar_arrive_expect_tx(bar, 2u * BOX_BYTES);
#pragma unroll
    for (int p = 0; p < 2; ++p)
        tc::tma_load_4d(sbase + OFF_U + p * 8192, &m.v, 64 * p, hi, t0, bi, bar);
}

// Arrivals that complete a "ready" barrier: one per compute warp (16) for
// R_P2, R_P5 and R_E, whose operands each warp writes for itself; eight for
// R_P4 and R_O (the warps that write them); one for R_OP, from compute thread
// 0 after a compute barrier (the state scales the operand pass leaves are
// read across warps right after it).
__host__ __device__ constexpr uint32_t ready_count(uint32_t id);

// Compute thread 0 waits on `bar`; the compute barrier that follows releases
// the other compute threads.
__device__ __forceinline__ void wait_then_sync(uint32_t bar, uint32_t parity, int tid,
                                               volatile int* abort_s) {
    if (tid == 0 && !*abort_s && !tc::mbar_wait_bounded(bar, parity, WAIT_NS)) *abort_s = 1;
    compute_sync();
    tc::fence_after_sync();
}

// Barriers (8 bytes each from OFF_BAR).  TMA arrivals and tensor-core
// commits complete the first group; the compute threads tell the issuing
// warp that an operand set is in place through the second (thread 0 arrives
// after a compute barrier; for R_O each of the 8 warps that write the o
// staging tile arrives once).
enum : uint32_t {
    B_KQW, B_AB, B_V,              // raw k, q, w / a, b / v landed
    B_G, B_XAU, B_E, B_ST, B_FIN,  // products done: gram / X, S~, A U / E / O, S~ / all
    R_OP, R_P2, R_P4, R_P5, R_E, R_O  // ready for: gram / X, S~ / A U / E / O, S~ / o store
};
static_assert(R_O + 1 == NBAR, "barrier count");
__host__ __device__ constexpr uint32_t ready_count(uint32_t id) {
    return (id == R_P2 || id == R_P5 || id == R_E) ? 16u : (id == R_P4 || id == R_O) ? 8u : 1u;
}

// PACKED: packed sequences (rows past a sequence's end are zeroed rather than
// left to the TMA fill).  FG2: FG^2-GDN learning rates among the gates.  DUMP:
// no o; instead every chunk's operand S~ = Diag(g_m) S0 (bf16, the tile its
// products read) goes through the sst map to slot bh * n_slots + slot0 +
// chunk of a [slots][128][128] array, and, when o_raw is given, each chunk's
// E (the key reads, bf16 [B, T, H, 128]) to o_raw through the o map: what
// the backward reads back.  All
// compile-time, so the plain instantiation carries none of these tests.
// T_row: tokens between batch rows in memory (T, or more when the launch
// covers a token range of longer rows).
template <bool PACKED, bool FG2, bool DUMP>
__global__ void __launch_bounds__(NT, 1)
chunked_tc_kernel(const __grid_constant__ TcMaps maps, int B, int T, int H,
                  const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                  const __nv_bfloat16* __restrict__ w, int a_kind, int b_kind, int w_kind,
                  const float* __restrict__ s0, float* __restrict__ s_final,
                  int* __restrict__ err_word, int skip_signal,
                  const int* __restrict__ cu_seqlens, __nv_bfloat16* __restrict__ o_raw,
                  int n_slots, int slot0, int T_row) {
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
    auto bar = [&](uint32_t id) { return sbase + OFF_BAR + 8u * id; };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quarter = warp & 3;                  // tensor-memory lanes 32*quarter ..
    const int cb = warp >> 2;                      // 32-column block this warp reads
    const int lane_t = 32 * quarter + (tid & 31);  // tensor-memory lane of this thread
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;

    const int bh = blockIdx.x;
    const int hi = bh % H;
    // this CTA's tokens: [tb, tb + L) of batch row bi (packed sequences: one
    // batch row; a range outside the tensor is reported and skipped)
    int bi, tb, L;
    if (!seq_range(cu_seqlens, bh / H, T, bi, tb, L)) {
        if (threadIdx.x == 0) atomicOr(err_word, kErrIndex);
        return;
    }
    const size_t soff = (size_t)bh * D * D;
    const bool fb = b_kind == GDR_GATE_FG2, fw = w_kind == GDR_GATE_FG2;
    const bool va = a_kind == GDR_GATE_VECTOR, vb = b_kind == GDR_GATE_VECTOR || fb,
               vw = w_kind == GDR_GATE_VECTOR || fw;
    const bool has_ab = va || vb;

    if (tid == 0) {
#pragma unroll 1
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(bar(i), ready_count(i));
        tc::mbar_fence_init();
        *abort_s = 0;
    }
    if (tid < D) fprev[tid] = 1.0f;
    // rows 64-127 of Z3 and the 16 x 16 blocks above the diagonal of T - I
    // (its rows 0-63) stay zero for the whole sequence
    if (tid < NTC) {
        const int r = tid >> 3, c16 = tid & 7;
        if ((c16 >> 1) > (r >> 4))
            *reinterpret_cast<uint4*>(sm + OFF_Z3 + r * 128 + ((c16 ^ (r & 7)) << 4)) =
                make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + OFF_Z3 + 8192 + 16 * tid) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (warp == 0) tc::tmem_alloc(sbase + OFF_TSLOT, 512);
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TSLOT);

    if (warp == NTC / 32) {
        // ======================= issuing warp (one thread)
        if ((tid & 31) == 0 && L > 0) {
            tc::tma_prefetch_desc(&maps.q);
            tc::tma_prefetch_desc(&maps.k);
            tc::tma_prefetch_desc(&maps.v);
            const bool dump_e = DUMP && o_raw != nullptr;
            if (!DUMP || dump_e) tc::tma_prefetch_desc(&maps.o);
            uint32_t ph = 0;               // phase of the per-chunk barriers
            uint32_t n_kqw = 0, n_ab = 0, n_v = 0;
            issue_kqw(maps, sbase, tb, hi, bi, vw, bar(B_KQW)); ++n_kqw;
            if (has_ab) { issue_ab(maps, sbase, tb, hi, bi, va, vb, bar(B_AB)); ++n_ab; }
            issue_v(maps, sbase, tb, hi, bi, bar(B_V)); ++n_v;
            auto wait_ready = [&](uint32_t id) {
                if (!tc::mbar_wait_bounded(bar(id), ph, WAIT_NS)) { *abort_s = 1; return false; }
                tc::fence_after_sync();
                return *abort_s == 0;
            };
            const uint32_t idKK = tc::idesc_bf16(128, 128, 0, 0);
            const uint32_t idKM = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t idMM = tc::idesc_bf16(128, 128, 1, 1);
            // o of the chunk before t0 leaves by TMA once its staging tile is written
            auto store_o = [&](int t0o, uint32_t parity) {
                if (!tc::mbar_wait_bounded(bar(R_O), parity, WAIT_NS)) { *abort_s = 1; return false; }
                tc::tma_store_4d(&maps.o, sbase + OFF_OST, 0, hi, tb + t0o, bi);
                tc::tma_store_4d(&maps.o, sbase + OFF_OST + 8192, 64, hi, tb + t0o, bi);
                tc::bulk_commit();
                return true;
            };
            int t0 = 0;
#pragma unroll 1
            for (; t0 < L; t0 += C, ph ^= 1) {
                const bool has_next = t0 + C < L;
                if (!DUMP && t0 > 0 && !store_o(t0 - C, ph ^ 1)) break;
                // operands of the chunk are in place
                if (!wait_ready(R_OP)) break;
                // gram [K';Q'] [K";B"]^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_G, tc::desc_kmajor(sbase + OFF_X1, 16384, kk),
                                 tc::desc_kmajor(sbase + OFF_X2, 16384, kk), idKK, kk > 0);
                tc::bulk_wait_read();  // the o store has left its staging tile (NS reuses it)
                // (test hook: the first gram's signal left out; the compute threads'
                // bounded wait for it runs out)
                if (!(skip_signal && t0 == 0)) tc::mma_commit(bar(B_G));
                // X = [K';Q'] S~, S~ += K"^T U
                if (!wait_ready(R_P2)) break;
                if (DUMP) {  // S~ leaves by TMA (read before this chunk's state update completes)
                    const int slot = bh * n_slots + slot0 + t0 / C;
                    tc::tma_store_4d(&maps.sst, sbase + OFF_S0, 0, 0, slot, 0);
                    tc::tma_store_4d(&maps.sst, sbase + OFF_S0 + 16384, 64, 0, slot, 0);
                    tc::bulk_commit();
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_X1, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_S0, 16384, kk), idKM, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_X2, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_U, 8192, kk), idMM, true);
                // X += [A_kk; A_qk] U
                if (!wait_ready(R_P4)) break;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16_ts(tmem + TM_X, tmem + TM_AQ + 8 * kk,
                                    tc::desc_mnmajor(sbase + OFF_U, 8192, kk), idKM, true);
                tc::mma_commit(bar(B_XAU));
                if (has_next) {
                    // the next chunk's raw tiles, issued under the UT solve (TMA issue
                    // is slow enough to keep off the products' path): RAW and W were
                    // consumed by the operand pass, X1 and U are free once these
                    // products are done
                    issue_kqw(maps, sbase, tb + t0 + C, hi, bi, vw, bar(B_KQW)); ++n_kqw;
                    if (!tc::mbar_wait_bounded(bar(B_XAU), ph, WAIT_NS)) { *abort_s = 1; break; }
                    if (has_ab) { issue_ab(maps, sbase, tb + t0 + C, hi, bi, va, vb, bar(B_AB)); ++n_ab; }
                    issue_v(maps, sbase, tb + t0 + C, hi, bi, bar(B_V)); ++n_v;
                }
                // X += [T - I; 0] R (rows 0-63 become E)
                if (!wait_ready(R_P5)) break;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_Z3, 8192, kk),
                                 tc::desc_mnmajor(sbase + OFF_X2, 16384, kk), idKM, true);
                tc::mma_commit(bar(B_E));
                // X += [0; -A_qb] E (rows 64-127 become O); S~ -= B"^T E
                if (!wait_ready(R_E)) break;
                if (DUMP) tc::bulk_wait_read();  // the S~ store has read its tile
                if (dump_e) {  // E leaves by TMA (its tile is next reused after the gram)
                    tc::tma_store_4d(&maps.o, sbase + OFF_EB, 0, hi, tb + t0, bi);
                    tc::tma_store_4d(&maps.o, sbase + OFF_EB + 8192, 64, hi, tb + t0, bi);
                    tc::bulk_commit();
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_X, tc::desc_kmajor(sbase + OFF_Z3 + 8192, 8192, kk),
                                 tc::desc_mnmajor(sbase + OFF_EB, 8192, kk), idKM, true);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_S, tc::desc_mnmajor(sbase + OFF_X2 + 8192, 16384, kk),
                                 tc::desc_mnmajor(sbase + OFF_EB, 8192, kk),
                                 idMM | IDESC_NEG_B, true);
                tc::mma_commit(bar(B_ST));
            }
            // the last chunk's o (packed sequences: written directly, the TMA box
            // would reach into the next sequence)
            if (!DUMP && t0 >= L && *abort_s == 0 && !cu_seqlens) store_o(t0 - C, ph ^ 1);
            // nothing of this CTA may still be in flight when it exits
            tc::mma_commit(bar(B_FIN));
            tc::mbar_wait_bounded(bar(B_FIN), 0, WAIT_NS);
            if (n_kqw) tc::mbar_wait_bounded(bar(B_KQW), (n_kqw - 1) & 1, WAIT_NS);
            if (n_ab) tc::mbar_wait_bounded(bar(B_AB), (n_ab - 1) & 1, WAIT_NS);
            if (n_v) tc::mbar_wait_bounded(bar(B_V), (n_v - 1) & 1, WAIT_NS);
            tc::bulk_wait_all();
        }
    } else {
        // ======================= compute warps
        // scalar gates of chunk starting at t0n into buffer `buf` (1.0 past T)
        auto load_scalars = [&](int t0n, int buf) {
            if (tid < C) {
                const int nn = min(C, L - t0n);
                const long long tok = ((long long)bi * T_row + tb + t0n + tid) * H + hi;
                const bool in = tid < nn;
                float* sc = sca_all + buf * 192;
                sc[tid] = (a_kind == GDR_GATE_SCALAR && in) ? to_f32(a[tok]) : 1.f;
                sc[64 + tid] = (b_kind == GDR_GATE_SCALAR && in) ? to_f32(b[tok]) : 1.f;
                sc[128 + tid] = (w_kind == GDR_GATE_SCALAR && in) ? to_f32(w[tok]) : 1.f;
            }
        };
        if (L > 0) load_scalars(0, 0);

        // ---- initial state S0 (unscaled) into tensor memory: lane i, columns j
        {
            const int c0 = 32 * cb;
            float vals[32];
            if (s0) {
                const float4* src =
                    reinterpret_cast<const float4*>(s0 + soff + (size_t)lane_t * D + c0);
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
            tc::tmem_st32(tmem + lane_off + TM_S + c0, vals);
            tc::tmem_wait_st();
        }
        compute_sync();   // the first chunk's scalar gates are in place
        uint32_t ph = 0;  // phase of the per-chunk barriers
        // O (rows 64-127 of X) -> bf16 staging tile, by the warps of lanes 64-127
        // (each such warp then signals R_O: the issuing warp stores o as soon as
        // all 8 have written)
        auto read_o = [&] {
            if (quarter >= 2) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float vals[16];
                    tc::tmem_ld16(tmem + lane_off + TM_X + 32 * cb + 16 * hh, vals);
                    tc::tmem_wait_ld();
                    tc::store_row16_bf16(sm + OFF_OST + (cb >> 1) * 8192, lane_t - 64,
                                         2 * (cb & 1) + hh, vals);
                }
                tc::fence_async_smem();
                __syncwarp();
                if ((tid & 31) == 0) tc::mbar_arrive(bar(R_O));
            }
        };
        // after the compute barrier that follows, thread 0 signals `id`
        auto signal = [&](uint32_t id) {
            compute_sync();
            if (tid == 0) tc::mbar_arrive(bar(id));
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
        for (int t0 = 0; t0 < L; t0 += C, ph ^= 1) {
            const bool has_next = t0 + C < L;
            const int cur = (t0 / C) & 1;
            const float* sca = sca_all + cur * 192;

            // ================= P1: the chunk's raw tiles; decay factors, scaled operands
            // every compute thread waits on the tile groups itself (no CTA
            // barrier here: the previous chunk ended on one); a wait that runs
            // out sets the abort flag, and the vote at the chunk's end stops
            // all threads together
            if (!*abort_s) {
                bool ok = tc::mbar_wait_bounded(bar(B_KQW), ph, WAIT_NS);
                ok = ok && (!has_ab || tc::mbar_wait_bounded(bar(B_AB), ph, WAIT_NS));
                ok = ok && tc::mbar_wait_bounded(bar(B_V), ph, WAIT_NS);
                if (!ok) *abort_s = 1;
            }
            // ================= P1c:
            // K' over raw a, Q' over raw b (X1), K" and B" into X2, U over raw v;
            // the state scales: fcur = fprev g_m, fprev = gamma_63 / g_m
            operand_pass<PACKED, FG2>(sm, op_tiles(), tid, va, vb, vw, fb, fw, a_kind,
                         min(C, L - t0), sca, QT, err_word, [&] {
                             if (t0 == 0) return;
                             // the last chunk's state update has read X2 and EB and
                             // finished its O: O -> staging tile for the issuing warp
                             wait_each(B_ST, ph ^ 1);
                             if (!DUMP) read_o();
                         },
                         [&](int i, float g_m, float g_c) {
                             fcur[i] = fprev[i] * g_m;
                             fprev[i] = g_c;
                         });
            tc::fence_async_smem();
            signal(R_OP);

            // ================= P2: S~ <- f_i S~ (lane i), bf16 copy to smem
            {
                const int c0 = 32 * cb;
                const float f = fcur[lane_t];
                float vals[32];
                tc::fence_after_sync();
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
            warp_signal(R_P2);

            // ================= P3: the X and S~ products run under the gram readout
            wait_each(B_G, ph);

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
                    // [A_kk; A_qk] -> tensor memory (A operand of the next product)
                    uint32_t packed[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        packed[x] = tc::pack_bf16x2(vals[2 * x], vals[2 * x + 1]);
                    tc::tmem_st16(tmem + lane_off + TM_AQ + 16 * (cb & 1), packed);
                    tc::tmem_wait_st();
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
            // ================= P5: the two column halves of the gram go their own ways.
            //   warps 8-15 (A_kb, A_qb): UT transform T = (I + A_kb)^{-1};
            //   warps 0-7 ([A_kk; A_qk] in tensor memory): X += [A_kk; A_qk] U, R -> bf16
            if (warp >= 8) {
                tc::fence_async_smem();
                half_sync(2);
                ut_solve<0>(NS, TS, PS, sm + OFF_Z3, tid - 256);
                tc::fence_async_smem();
            } else {
                tc::fence_before_sync();
                warp_signal(R_P4);
                wait_each(B_XAU, ph);
                if (quarter < 2) {   // lanes 0-63 of X hold R; each warp takes 64 columns
                    const int c0 = 64 * cb;
                    float vals[32];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        tc::tmem_ld32(tmem + lane_off + TM_X + c0 + 32 * hh, vals);
                        tc::tmem_wait_ld();
                        // into the K" rows of X2, read by now
                        tc::store_row32_bf16(sm + OFF_X2 + (c0 >> 6) * 16384, lane_t, hh, vals);
                    }
                }
                tc::fence_async_smem();
                // the next chunk's scalar gates: these warps wait out the global
                // loads' latency under the solve
                if (has_next) load_scalars(t0 + C, cur ^ 1);
            }
            tc::fence_before_sync();
            warp_signal(R_P5);

            // ================= P6: X += [T - I; 0] R (rows 0-63 become E)
            wait_each(B_E, ph);

            // ================= P7: E -> bf16; X += [0; -A_qb] E and S~ -= B"^T E run
            // under the next chunk's decay products
            if (quarter < 2) {
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_X + 32 * cb, vals);
                tc::tmem_wait_ld();
                tc::store_row32_bf16(sm + OFF_EB + (cb >> 1) * 8192, lane_t, cb & 1, vals);
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            warp_signal(R_E);
            if (compute_sync_or(*abort_s != 0)) break;
        }
        // (one vote, so that all compute threads agree on whether to finish)
        if (L > 0 && !compute_sync_or(*abort_s != 0)) {
            // the last chunk's O
            wait_then_sync(bar(B_ST), ph ^ 1, tid, abort_s);
            if (DUMP) {
                // no outputs
            } else if (!cu_seqlens) {
                read_o();
            } else if (quarter >= 2) {
                // straight to global memory, only the sequence's own rows
                const int t0l = ((L - 1) / C) * C, r = lane_t - 64;
                float vals[32];
                tc::tmem_ld32(tmem + lane_off + TM_X + 32 * cb, vals);
                tc::tmem_wait_ld();
                if (r < L - t0l) {
                    uint4* dst = reinterpret_cast<uint4*>(
                        o_raw + (((long long)bi * T + tb + t0l + r) * H + hi) * D + 32 * cb);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 u;
                        u.x = tc::pack_bf16x2(vals[8 * x], vals[8 * x + 1]);
                        u.y = tc::pack_bf16x2(vals[8 * x + 2], vals[8 * x + 3]);
                        u.z = tc::pack_bf16x2(vals[8 * x + 4], vals[8 * x + 5]);
                        u.w = tc::pack_bf16x2(vals[8 * x + 6], vals[8 * x + 7]);
                        dst[x] = u;
                    }
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (*abort_s) {
        atomicOr(err_word, kErrTimeout);
    } else if (s_final && tid < NTC) {
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
bool make_map(CUtensorMap* m, const void* ptr, int B, int T, int H, int T_row) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                                   (cuuint64_t)T_row * H * D * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

// [B, T, H, 128] bf16 tensor map of the kernels' operand format (used by the
// backward's kernel too).
bool tc_map_bf16(CUtensorMap* m, const void* ptr, int B, int T, int H, int T_row) {
    return make_map(m, ptr, B, T, H, T_row);
}

// [B, T, H, 128] bf16 tensor as a 4-D map {128, H, T, B}, box {32, 1, 32, 1}
// (32 channels of 32 tokens, 64-byte rows), 64-byte swizzle: the backward's
// staging format for its intermediate outputs.
bool tc_map_bf16_box32(CUtensorMap* m, const void* ptr, int B, int T, int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                                   (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {32, 1, 32, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// [n_slots][128][128] bf16 state tiles (row = key channel) as a 4-D map
// {128, 128, n_slots, 1}, box {64, 128, 1, 1} (one 64-column panel of a
// tile), 128-byte swizzle: the operand layout of S~.
bool tc_map_state_bf16(CUtensorMap* m, const void* ptr, long long n_slots) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)D, (cuuint64_t)n_slots, 1};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)D * D * 2,
                                   (cuuint64_t)n_slots * D * D * 2};
    const cuuint32_t box[4] = {64, 128, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool chunked_tc_supports(const gdr_desc& d) {
    return d.in_dtype == GDR_BF16 && d.dk == D && d.dv == D && d.chunk == C;
}

namespace {
// Tensor maps of one launch; o only when it is written.
bool make_maps(TcMaps* maps, const gdr_desc& d, int T_row, const void* q, const void* k,
               const void* v, const void* a, const void* b, const void* w, const void* o) {
    memset(maps, 0, sizeof(*maps));
    if (d.T == 0) return true;
    const int B = d.B, T = d.T, H = d.H;
    bool ok = make_map(&maps->q, q, B, T, H, T_row) && make_map(&maps->k, k, B, T, H, T_row) &&
              make_map(&maps->v, v, B, T, H, T_row);
    if (ok && o) ok = make_map(&maps->o, o, B, T, H, T_row);
    if (ok && d.decay == GDR_GATE_VECTOR) ok = make_map(&maps->a, a, B, T, H, T_row);
    if (ok && (d.erase == GDR_GATE_VECTOR || d.erase == GDR_GATE_FG2))
        ok = make_map(&maps->b, b, B, T, H, T_row);
    if (ok && (d.write == GDR_GATE_VECTOR || d.write == GDR_GATE_FG2))
        ok = make_map(&maps->w, w, B, T, H, T_row);
    return ok;
}
}  // namespace

cudaError_t launch_chunked_tc(const gdr_desc& d, const void* q, const void* k, const void* v,
                              const void* a, const void* b, const void* w, const float* s0,
                              void* o, float* s_final, int* err_word, bool skip_signal,
                              const int* cu_seqlens, int n_seqs, cudaStream_t st) {
    TcMaps maps;
    if (!make_maps(&maps, d, d.T, q, k, v, a, b, w, o)) return cudaErrorInvalidValue;
    const bool fg2 = d.erase == GDR_GATE_FG2 || d.write == GDR_GATE_FG2;
    auto kern = cu_seqlens
                    ? (fg2 ? chunked_tc_kernel<true, true, false> : chunked_tc_kernel<true, false, false>)
                    : (fg2 ? chunked_tc_kernel<false, true, false> : chunked_tc_kernel<false, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long nseq = cu_seqlens ? n_seqs : d.B;
    kern<<<(unsigned)(nseq * d.H), NT, SMEM_BYTES, st>>>(
        maps, d.B, d.T, d.H, (const __nv_bfloat16*)a, (const __nv_bfloat16*)b,
        (const __nv_bfloat16*)w, (int)d.decay, (int)d.erase, (int)d.write, s0, s_final,
        err_word, skip_signal ? 1 : 0, cu_seqlens, (__nv_bfloat16*)o, 0, 0, d.T);
    return cudaGetLastError();
}

// Every 64-token chunk's S~ = Diag(g_m) S0 of the B x H sequences (no o), as
// bf16 into slots slot0, slot0 + 1, ... of `s_tilde` ([B*H][n_slots][128][128],
// row = key channel), and, if e_out is given, every chunk's E (bf16
// [B, T, H, 128]): what the backward reads back.  The launch covers d.T
// tokens of rows T_row tokens apart (the pointers already at its first
// token); s_final, if given, receives the state after them.
cudaError_t launch_chunked_tc_states(const gdr_desc& d, int T_row, const void* q, const void* k,
                                     const void* v, const void* a, const void* b,
                                     const void* w, const float* s0, float* s_final,
                                     void* s_tilde, int n_slots, int slot0, void* e_out,
                                     int* err_word, cudaStream_t st) {
    TcMaps maps;
    if (!make_maps(&maps, d, T_row, q, k, v, a, b, w, e_out)) return cudaErrorInvalidValue;
    if (d.T > 0 && !tc_map_state_bf16(&maps.sst, s_tilde, (long long)d.B * d.H * n_slots))
        return cudaErrorInvalidValue;
    const bool fg2 = d.erase == GDR_GATE_FG2 || d.write == GDR_GATE_FG2;
    auto kern = fg2 ? chunked_tc_kernel<false, true, true> : chunked_tc_kernel<false, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((long long)d.B * d.H), NT, SMEM_BYTES, st>>>(
        maps, d.B, d.T, d.H, (const __nv_bfloat16*)a, (const __nv_bfloat16*)b,
        (const __nv_bfloat16*)w, (int)d.decay, (int)d.erase, (int)d.write, s0, s_final,
        err_word, 0, nullptr, (__nv_bfloat16*)e_out, n_slots, slot0, T_row);
    return cudaGetLastError();
}

}  // namespace gdr
