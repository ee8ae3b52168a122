// backward.cu -- gradients of the chunked gated delta rule for the cases the
// tcgen05 backward (bwd_tc.cu: bf16, dk = dv = 128, one sequence per batch
// row) does not take: float32 inputs (products on the CUDA cores in
// float32), head dimension 64 and packed sequences (bf16: products on the
// tensor cores as mma.sync with tf32 operands, float32 accumulation).
//
// Loss L = sum_t <o_t, do_t> + <S_T, dS_T>; the kernel returns dL/dq, dk, dv,
// the three gates and dS_0.  The pages train the recurrence in its chunked
// form (FG^2-GDN page, gist.science 2604.19021, section 2 "Methodology": the
// rank-1 Householder structure kept for WY chunked training); the gradient
// identities below are the reverse of the chunked forward, derived here.
//
// Forward of one chunk (n <= C tokens, state S0 at its start; G_r = sum of
// log a over tokens 0..r of the chunk, per key channel; G_C = G_{n-1}):
//   Qh = e^G q, Kh = e^G k, Kt = e^(G_C - G) k, Bt = b Kt, U = w v
//   A_qk = tril(Qh Kb^T), A_qb = tril(Qh Bb^T)          (s <= r)
//   A_kk = tril(Kh Kb^T), A_kb = tril(Kh Bb^T)          (s <  r)
//     with Kb = e^-G_C Kt = e^-G k, Bb = e^-G_C Bt
//   Y = Kh S0 + A_kk U,  E = T Y,  T = (I + A_kb)^-1    (row r of E: the key
//                                                        read e_r of token r)
//   O = Qh S0 + A_qk U - A_qb E
//   S_C = e^G_C S0 + Kt^T U - Bt^T E
// Reverse, given dO and dS_C:
//   dE = -A_qb^T dO - Bt dS_C,   dY = T^T dE
//   dU = A_qk^T dO + A_kk^T dY + Kt dS_C
//   dA_qk = dO U^T, dA_qb = -dO E^T, dA_kk = dY U^T, dA_kb = -dY E^T  (masked)
//   dS0 = e^G_C dS_C + Qh^T dO + Kh^T dY                (dS_C of the chunk before)
//   XQ = dQh = dO S0^T + e^-G_C (dA_qk Kt + dA_qb Bt)
//   XK = dKh = dY S0^T + e^-G_C (dA_kk Kt + dA_kb Bt)
//   YK = U dS_C^T + e^-G_C (dA_qk^T Qh + dA_kk^T Kh)     (gradient on Kt, with the
//   YB = -E dS_C^T + e^-G_C (dA_qb^T Qh + dA_kb^T Kh)     grams' share folded in)
//   dq = e^G XQ,  dk = e^G XK + e^(G_C - G) (YK + b YB),  db = Kt YB
//   dv = w dU,  dw = v dU
//   dG = Qh XQ + Kh XK - Kt YK - Bt YB, plus at row n-1
//        e^G_C rowsum(dS_C * S0) + colsum(Kt * U dS_C^T - Bt * E dS_C^T)
//   d log a_r = sum_{r' >= r} dG_r',  da = d log a / a
//
// Range: the factors e^-G_C reach e^80 at most when every channel's decay over
// a chunk multiplies to at least e^-80; a chunk below that is reported
// (GDR_ERR_RANGE) like the tensor-core forward's range check.
//
// FG^2-GDN learning rates (gate kind FG2; FG^2-GDN page, section 2): the key
// used is sqrt(beta^k) k with erase gate 1, the write gate sqrt(beta^v).  The
// gradients above are taken for that key and write gate, then carried
// through the square roots: dk = sqrt(beta^k) dk~, dbeta^k = k dk~ /
// (2 sqrt(beta^k)), dbeta^v = v dU / (2 sqrt(beta^v)) (beta > 0).
//
// Packed sequences (cu_seqlens): CTA (sequence, head) takes its sequence's
// tokens; its chunk-start states follow those of the sequences before it.
//
// One launch, one CTA per (batch, head).  A forward sweep first stores the
// state at the start of every chunk in the workspace (the chunk form above
// without its outputs); the reverse sweep then walks the chunks backwards,
// carrying dS in the workspace (L2-resident, one [dk, dv] matrix per head).
// Per chunk: stage A forms the gated operands, the grams and T; stage B runs
// the value-side products in blocks of 16 columns, keeping dA and the
// [C, dk] gradient sums in registers; stage C adds the grams' gradients;
// stage D maps the sums back to q, k, b and the decay.  On the CUDA cores the
// products are register tiles fed by 16-byte shared-memory loads (rows of the
// [*, dk] tiles are float4-aligned), with the state blocks held transposed
// ([value column][key channel]) so both operands of the key-side sums load
// as float4.  On the tensor cores each warp owns 16 x 8 output tiles and reads
// its fragments from the same float32 tiles.
#include "common.cuh"

namespace gdr {

constexpr int BW_C = 32;    // tokens per chunk
constexpr int BW_DB = 16;   // value columns per stage-B block
constexpr int BW_NT = 512;  // threads
constexpr float BW_MIN_LOG_DECAY = -80.0f;

template <int DK>
struct BwdSmem {
    static constexpr int C = BW_C, DB = BW_DB;
    static constexpr int P = DK + 4;   // row stride of [C][DK] and [DB][DK] tiles
    static constexpr int CP = C + 1;   // row stride of [C][C] tiles
    static constexpr int UP = DB + 4;  // row stride of [C][DB] tiles
    static constexpr int kQh = 0;
    static constexpr int kKh = kQh + C * P;
    static constexpr int kKt = kKh + C * P;
    static constexpr int kBt = kKt + C * P;
    static constexpr int kB = kBt + C * P;  // erase gate
    static constexpr int kG = kB + C * P;   // cumulative log decay
    static constexpr int kA = kG + C * P;   // decay a itself (for da = d log a / a)
    static constexpr int kAqk = kA + C * P;
    static constexpr int kAqb = kAqk + C * CP;
    static constexpr int kAkk = kAqb + C * CP;
    static constexpr int kAkb = kAkk + C * CP;
    static constexpr int kT = kAkb + C * CP;
    static constexpr int kScr = kT + C * CP;
    // stage B tiles inside the scratch
    static constexpr int sS0 = 0;               // S0 block, [DB][DK]
    static constexpr int sdS = sS0 + DB * P;    // dS_C block, [DB][DK]
    static constexpr int sU = sdS + DB * P;
    static constexpr int sdO = sU + C * UP;
    static constexpr int sY = sdO + C * UP;
    static constexpr int sE = sY + C * UP;
    static constexpr int sdE = sE + C * UP;
    static constexpr int sdY = sdE + C * UP;
    static constexpr int scrB = sdY + C * UP;
    // stage D: dG [C][P]
    static constexpr int scrD = C * P;
    static constexpr int scr = ((scrB > scrD ? scrB : scrD) + 3) / 4 * 4;
    static constexpr int kGcr = kScr + scr;     // per-row shares of the G_C gradient [C][P]
    static constexpr int kDA = kGcr + C * P;    // dA_qk, dA_qb, dA_kk, dA_kb [C][CP] each
    static constexpr int kEgc = kDA + 4 * C * CP;  // e^G_C per channel
    static constexpr int kIgc = kEgc + DK;      // e^-G_C
    static constexpr int kDgc = kIgc + DK;      // gradient on G_C
    static constexpr int kDwp = kDgc + DK;     // scalar write gate: row sums per column half [2][C]
    static constexpr int floats = kDwp + 2 * C;
    static constexpr size_t bytes = sizeof(float) * floats;
    static_assert(kScr % 4 == 0 && kGcr % 4 == 0 && kEgc % 4 == 0 && sU % 4 == 0 &&
                  kDA % 4 == 0 &&
                  C * P % 4 == 0 && C * UP % 4 == 0, "float4 alignment");
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
// a . b added into two partial sums (even and odd components): two
// independent FMA chains instead of one four-deep chain.
__device__ __forceinline__ void dot4_2(float4 a, float4 b, float& e, float& o) {
    e = fmaf(a.x, b.x, e);
    o = fmaf(a.y, b.y, o);
    e = fmaf(a.z, b.z, e);
    o = fmaf(a.w, b.w, o);
}
// Tensor-core products of the bf16 path: mma.sync m16n8k8 with tf32 operands
// (round to nearest) and float32 accumulation, operands read straight from the
// float32 tiles in shared memory.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// One warp: acc (the 16 x 8 tile at rows m0, columns n0) += sum over k in
// [k0, k0 + K) of A(m, k) B(k, n).  A(m, k) = A[m * lda + k], or A[k * lda + m]
// when AT; B(k, n) = B[k * ldb + n] when BK (stored [K][N]), else B[n * ldb + k].
// Lane (g = lane / 4, t = lane % 4) holds D(m0 + g, n0 + 2t), D(m0 + g, n0 + 2t + 1),
// D(m0 + g + 8, n0 + 2t), D(m0 + g + 8, n0 + 2t + 1) in acc[0..3]; K is a multiple of 8.
// With ks, B(k, n) is also multiplied by ks[k].
template <bool AT, bool BK>
__device__ __forceinline__ void mma_tile(float (&acc)[4], const float* A, int lda, const float* B,
                                         int ldb, int m0, int n0, int k0, int K,
                                         const float* ks = nullptr) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    auto ea = [&](int m, int kk) { return AT ? A[kk * lda + m] : A[m * lda + kk]; };
    auto eb = [&](int kk, int nn) {
        const float x = BK ? B[kk * ldb + nn] : B[nn * ldb + kk];
        return ks ? x * ks[kk] : x;
    };
#pragma unroll 4
    for (int k = k0; k < k0 + K; k += 8) {
        uint32_t a[4];
        a[0] = to_tf32(ea(m0 + g, k + t));
        a[1] = to_tf32(ea(m0 + g + 8, k + t));
        a[2] = to_tf32(ea(m0 + g, k + t + 4));
        a[3] = to_tf32(ea(m0 + g + 8, k + t + 4));
        mma_tf32(acc, a, to_tf32(eb(k + t, n0 + g)), to_tf32(eb(k + t + 4, n0 + g)));
    }
}
// Element x of a lane's tile: row m0 + g + 8 (x >> 1), column n0 + 2t + (x & 1).
__device__ __forceinline__ int tile_row(int m0, int x) { return m0 + ((threadIdx.x & 31) >> 2) + 8 * (x >> 1); }
__device__ __forceinline__ int tile_col(int n0, int x) { return n0 + 2 * (threadIdx.x & 3) + (x & 1); }
__device__ __forceinline__ void store_tile(float* dst, int ld, int m0, int n0, const float (&acc)[4],
                                           float sign = 1.f) {
#pragma unroll
    for (int x = 0; x < 4; ++x) dst[tile_row(m0, x) * ld + tile_col(n0, x)] = sign * acc[x];
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}

__device__ __forceinline__ float comp(float4 v, int e) {
    return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}

// Four consecutive values of a gradient row (16-byte or 8-byte store).
__device__ __forceinline__ void store4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
}

// MMA: the products on the tensor cores (tf32, bf16 inputs); otherwise on the
// CUDA cores in float32 (float32 inputs and their 1e-4 budget).
template <typename Tin, int DK, int DV, bool MMA>
__global__ void __launch_bounds__(BW_NT, 1)
backward_kernel(int T, int H, const int* __restrict__ cu_seqlens,
                const Tin* __restrict__ q, const Tin* __restrict__ k,
                const Tin* __restrict__ v, const Tin* __restrict__ a,
                const Tin* __restrict__ b, const Tin* __restrict__ w, int a_kind, int b_kind,
                int w_kind, const Tin* __restrict__ dout, const float* __restrict__ s0,
                const float* __restrict__ ds_final, float* __restrict__ hs,
                float* __restrict__ ds_run, Tin* __restrict__ dq, Tin* __restrict__ dk,
                Tin* __restrict__ dv, Tin* __restrict__ da, Tin* __restrict__ db,
                Tin* __restrict__ dw, float* __restrict__ ds0, int* __restrict__ err_word) {
    using L = BwdSmem<DK>;
    constexpr int C = BW_C, DB = BW_DB, NT = BW_NT;
    constexpr int P = L::P, CP = L::CP, UP = L::UP;
    constexpr int NG = DK / 64;      // float4 groups of key channels per thread: 4 cl + 64 g
    constexpr int NCI = 4 * NG;      // key channels per thread in the [C][DK] sums
    static_assert(C * DB == NT && DV % DB == 0 && (DK == 64 || DK == 128), "shape");

    extern __shared__ __align__(16) float sm[];
    float* Qh = sm + L::kQh;
    float* Kh = sm + L::kKh;
    float* Kt = sm + L::kKt;
    float* Bt = sm + L::kBt;
    float* Bs = sm + L::kB;
    float* Gs = sm + L::kG;
    float* As = sm + L::kA;
    float* Aqk = sm + L::kAqk;
    float* Aqb = sm + L::kAqb;
    float* Akk = sm + L::kAkk;
    float* Akb = sm + L::kAkb;
    float* Tm = sm + L::kT;
    float* scr = sm + L::kScr;
    float* S0T = scr + L::sS0;
    float* dST = scr + L::sdS;
    float* Ub = scr + L::sU;
    float* dOb = scr + L::sdO;
    float* Yb = scr + L::sY;
    float* Eb = scr + L::sE;
    float* dEb = scr + L::sdE;
    float* dYb = scr + L::sdY;
    float* gcr = sm + L::kGcr;
    float* dAqk = sm + L::kDA;
    float* dAqb = dAqk + C * CP;
    float* dAkk = dAqk + 2 * C * CP;
    float* dAkb = dAqk + 3 * C * CP;
    float* egc = sm + L::kEgc;
    float* igc = sm + L::kIgc;
    float* dgc = sm + L::kDgc;
    float* dwp = sm + L::kDwp;

    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int seq = bh / H, hi = bh % H;
    // this CTA's tokens: [tb, tb + len) of batch row bi.  Packed sequences must
    // be ordered (cu non-decreasing from cu[0] >= 0 up to this one): that bounds
    // the chunk-state offset below by the workspace size; otherwise the
    // sequence is reported and skipped.
    int bi, tb, len;
    long long chunk_base = 0;  // chunk-start states of the sequences before this one
    bool ok = seq_range(cu_seqlens, seq, T, bi, tb, len);
    if (cu_seqlens) {
        ok = ok && cu_seqlens[0] >= 0;
        for (int m = 0; ok && m < seq; ++m) {
            const int l = cu_seqlens[m + 1] - cu_seqlens[m];
            ok = l >= 0;
            chunk_base += (l + BW_C - 1) / BW_C;
        }
    } else {
        chunk_base = (long long)seq * ((T + BW_C - 1) / BW_C);
    }
    if (!ok) {
        if (tid == 0 && hi == 0) atomicOr(err_word, kErrIndex);
        return;
    }
    const int rr = tid >> 4;   // row in [C][*] tiles (one row per thread)
    const int cl = tid & 15;   // lane in the row: value column, or key channels 4 cl + 64 g
    const int task = tid >> 8; // two half-CTA tasks side by side in stage B
    const int t2 = tid & 255;
    const int r2 = t2 >> 4;    // rows r2 and r2 + 16 of a half-CTA task
    const int n_chunks = (len + C - 1) / C;
    const size_t soff = (size_t)bh * DK * DV;
    float* hbase = hs + ((size_t)chunk_base * H + (size_t)hi * n_chunks) * DK * DV;
    auto tok_of = [&](int t) { return ((long long)bi * T + tb + t) * H + hi; };
    const bool fg2_b = b_kind == GDR_GATE_FG2;

    // ---------------- stage A: gated operands, grams (all four when with_q), T
    auto stage_a = [&](int t0, int n, bool with_q) {
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f, av = 1.f;
            if (r < n) {
                const long long tok = tok_of(t0 + r), base = tok * DK;
                if (with_q) qv = to_f32(q[base + c]);
                kv = to_f32(k[base + c]);
                bv = gate_value(b, b_kind, tok, base, c);  // FG2: sqrt(beta^k)
                if (fg2_b) kv *= bv;                       // key sqrt(beta^k) k, erase gate 1
                av = gate_value(a, a_kind, tok, base, c);
                gv = a_kind == GDR_GATE_ONE ? 0.f : safe_log_decay(av);
            }
            Qh[r * P + c] = qv;
            Kh[r * P + c] = kv;
            Bs[r * P + c] = bv;
            Gs[r * P + c] = gv;
            As[r * P + c] = av;
        }
        __syncthreads();
        if (tid < DK) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                run += Gs[r * P + tid];
                Gs[r * P + tid] = run;
            }
            if (run < BW_MIN_LOG_DECAY) atomicOr(err_word, kErrRange);
            egc[tid] = __expf(run);
            igc[tid] = __expf(-run);
        }
        __syncthreads();
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            const float g = Gs[r * P + c], gc = Gs[(C - 1) * P + c];
            const float eg = __expf(g), et = __expf(gc - g);
            const float kv = Kh[r * P + c];
            Qh[r * P + c] *= eg;
            Kh[r * P + c] = kv * eg;
            Kt[r * P + c] = kv * et;
            Bt[r * P + c] = (fg2_b ? 1.f : Bs[r * P + c]) * kv * et;
        }
        __syncthreads();
        if constexpr (MMA) {  // grams on the tensor cores: 4 x (2 x 4) tiles, two per warp
            const int wid = tid >> 5;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int id = 2 * wid + u, mat = id >> 3, rem = id & 7;  // qk, qb, kk, kb
                if (!with_q && mat < 2) continue;
                const int m0 = 16 * (rem >> 2), n0 = 8 * (rem & 3);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                // A(r, c) = Qh or Kh; B(c, s) = e^-G_C[c] Kt[s][c] or e^-G_C[c] Bt[s][c]
                mma_tile<false, false>(acc, mat < 2 ? Qh : Kh, P, (mat & 1) ? Bt : Kt, P, m0, n0,
                                       0, DK, igc);
                float* dst = mat == 0 ? Aqk : mat == 1 ? Aqb : mat == 2 ? Akk : Akb;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int r = tile_row(m0, x), sc = tile_col(n0, x);
                    const bool keep = mat < 2 ? sc <= r : sc < r;
                    dst[r * CP + sc] = keep ? acc[x] : 0.f;
                }
            }
        } else {
            const int r = rr;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int s = cl + 16 * h2;
                float qk = 0.f, qb = 0.f, kk = 0.f, kb = 0.f;
                float qk2 = 0.f, qb2 = 0.f, kk2 = 0.f, kb2 = 0.f;
                if (s <= r) {
#pragma unroll 4
                    for (int c = 0; c < DK; c += 4) {
                        const float4 ig = ld4(igc + c);
                        float4 kb4 = ld4(Kt + s * P + c), bb4 = ld4(Bt + s * P + c);
                        kb4.x *= ig.x; kb4.y *= ig.y; kb4.z *= ig.z; kb4.w *= ig.w;
                        bb4.x *= ig.x; bb4.y *= ig.y; bb4.z *= ig.z; bb4.w *= ig.w;
                        const float4 kr = ld4(Kh + r * P + c);
                        dot4_2(kr, kb4, kk, kk2);
                        dot4_2(kr, bb4, kb, kb2);
                        if (with_q) {
                            const float4 qr = ld4(Qh + r * P + c);
                            dot4_2(qr, kb4, qk, qk2);
                            dot4_2(qr, bb4, qb, qb2);
                        }
                    }
                }
                kk += kk2;
                kb += kb2;
                qk += qk2;
                qb += qb2;
                Akk[r * CP + s] = s < r ? kk : 0.f;
                Akb[r * CP + s] = s < r ? kb : 0.f;
                if (with_q) {
                    Aqk[r * CP + s] = qk;
                    Aqb[r * CP + s] = qb;
                }
            }
        }
        __syncthreads();
        // T = (I + N)^-1, N = A_kb strictly lower (C = 32), by 16 x 16 blocks:
        // the diagonal blocks by substitution (thread = column of one of
        // them: at most 120 steps instead of 496 for a column of T), then
        // T21 = -T22 N21 T11 (two 16 x 16 products, one output per thread);
        // T12 = 0.  The scratch region is free during stage A.
        static_assert(C == 32 && NT >= 256, "blocked inverse shape");
        if (tid < 32) {
            const int o = 16 * (tid >> 4), c = tid & 15;
#pragma unroll 1
            for (int r = 0; r < 16; ++r) {   // column c of the diagonal block at o
                float t = (r == c) ? 1.f : 0.f;
#pragma unroll 1
                for (int s2 = c; s2 < r; ++s2)   // entries above row c are zero
                    t = fmaf(-Akb[(o + r) * CP + o + s2], Tm[(o + s2) * CP + o + c], t);
                Tm[(o + r) * CP + o + c] = t;
                if (o == 0) Tm[r * CP + 16 + c] = 0.f;
            }
        }
        __syncthreads();
        float* ys = scr;  // Y = N21 T11, 16 x 16
        if (tid < 256) {
            const int r = tid >> 4, c = tid & 15;
            float acc = 0.f;
#pragma unroll 1
            for (int s2 = c; s2 < 16; ++s2)  // T11 is lower triangular
                acc = fmaf(Akb[(16 + r) * CP + s2], Tm[s2 * CP + c], acc);
            ys[r * 16 + c] = acc;
        }
        __syncthreads();
        if (tid < 256) {
            const int r = tid >> 4, c = tid & 15;
            float acc = 0.f;
#pragma unroll 1
            for (int s2 = 0; s2 <= r; ++s2)  // T22 is lower triangular
                acc = fmaf(Tm[(16 + r) * CP + 16 + s2], ys[s2 * 16 + c], acc);
            Tm[(16 + r) * CP + c] = -acc;
        }
        __syncthreads();
    };

    // The [DK][DB] block at column j0 of a [DK][DV] matrix, fetched into
    // registers ahead of its use and stored transposed ([DB][DK]) after the
    // barrier that frees the tile.
    constexpr int NPF = DK * DB / NT;
    auto fetch_block = [&](float (&reg)[NPF], const float* src, int j0) {
#pragma unroll
        for (int i = 0; i < NPF; ++i) {
            const int x = tid + NT * i, c = x / DB, j = x % DB;
            reg[i] = src[(size_t)c * DV + j0 + j];
        }
    };
    auto put_block = [&](float* dst, const float (&reg)[NPF]) {
#pragma unroll
        for (int i = 0; i < NPF; ++i) {
            const int x = tid + NT * i, c = x / DB, j = x % DB;
            dst[j * P + c] = reg[i];
        }
    };

    // ================= forward sweep: chunk-start states h_c into the workspace
    for (int x = tid; x < DK * DV; x += NT) {
        if (n_chunks > 0) hbase[x] = s0 ? s0[soff + x] : 0.f;
        ds_run[soff + x] = ds_final ? ds_final[soff + x] : 0.f;
    }
    // the state at the start of chunk ci + 1 from the one of chunk ci (a full chunk)
    auto fwd_step = [&](int ci) {
        const int t0 = ci * C;
        __syncthreads();  // h_ci written
        stage_a(t0, C, false);
        const float* hc = hbase + (size_t)ci * DK * DV;
        float* hn = hbase + (size_t)(ci + 1) * DK * DV;
        if constexpr (!MMA) {
        float pf_s[NPF];
        fetch_block(pf_s, hc, 0);
        for (int j0 = 0; j0 < DV; j0 += DB) {
            put_block(S0T, pf_s);
            {
                const long long tok = tok_of(t0 + rr), base = tok * DV;
                Ub[rr * UP + cl] = gate_value(w, w_kind, tok, base, j0 + cl) *
                                   to_f32(v[base + j0 + cl]);
            }
            __syncthreads();
            {  // Y = Kh S0 + A_kk U
                const int r = rr, j = cl;
                float y = 0.f, y2 = 0.f;
#pragma unroll 4
                for (int c = 0; c < DK; c += 4) dot4_2(ld4(Kh + r * P + c), ld4(S0T + j * P + c), y, y2);
                y += y2;
                for (int s = 0; s < r; ++s) y = fmaf(Akk[r * CP + s], Ub[s * UP + j], y);
                Yb[r * UP + j] = y;
            }
            __syncthreads();
            {  // E = T Y
                const int r = rr, j = cl;
                float e = 0.f;
                for (int s = 0; s <= r; ++s) e = fmaf(Tm[r * CP + s], Yb[s * UP + j], e);
                Eb[r * UP + j] = e;
            }
            __syncthreads();
            if (rr < DK / 4) {  // S_C = e^G_C S0 + Kt^T U - Bt^T E, channels 4 rr .. 4 rr + 3
                const int c = 4 * rr, j = cl;
                const float4 g4 = ld4(egc + c), s4 = ld4(S0T + j * P + c);
                float acc[4] = {g4.x * s4.x, g4.y * s4.y, g4.z * s4.z, g4.w * s4.w};
#pragma unroll 4
                for (int r = 0; r < C; ++r) {
                    const float4 kt = ld4(Kt + r * P + c), bt = ld4(Bt + r * P + c);
                    const float u = Ub[r * UP + j], e = Eb[r * UP + j];
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        acc[x] = fmaf(comp(kt, x), u, fmaf(-comp(bt, x), e, acc[x]));
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) hn[(size_t)(c + x) * DV + j0 + j] = acc[x];
            }
            if (j0 + DB < DV) fetch_block(pf_s, hc, j0 + DB);
            __syncthreads();  // block's tiles consumed
        }
        } else {
        float pf_s[NPF];
        fetch_block(pf_s, hc, 0);
        const int wid = tid >> 5;
        for (int j0 = 0; j0 < DV; j0 += DB) {
            put_block(S0T, pf_s);
            {
                const long long tok = tok_of(t0 + rr), base = tok * DV;
                Ub[rr * UP + cl] = gate_value(w, w_kind, tok, base, j0 + cl) *
                                   to_f32(v[base + j0 + cl]);
            }
            __syncthreads();
            if (wid < 4) {  // Y = Kh S0 + A_kk U: four 16 x 8 tiles
                const int m0 = 16 * (wid >> 1), n0 = 8 * (wid & 1);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tile<false, false>(acc, Kh, P, S0T, P, m0, n0, 0, DK);
                mma_tile<false, true>(acc, Akk, CP, Ub, UP, m0, n0, 0, C);
                store_tile(Yb, UP, m0, n0, acc);
            }
            __syncthreads();
            if (wid < 4) {  // E = T Y
                const int m0 = 16 * (wid >> 1), n0 = 8 * (wid & 1);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tile<false, true>(acc, Tm, CP, Yb, UP, m0, n0, 0, C);
                store_tile(Eb, UP, m0, n0, acc);
            }
            __syncthreads();
            if (wid < DK / 8) {  // S_C = e^G_C S0 + Kt^T U - Bt^T E: [DK][DB] in 16 x 8 tiles
                const int m0 = 16 * (wid >> 1), n0 = 8 * (wid & 1);
                float au[4] = {0.f, 0.f, 0.f, 0.f}, ae[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tile<true, true>(au, Kt, P, Ub, UP, m0, n0, 0, C);
                mma_tile<true, true>(ae, Bt, P, Eb, UP, m0, n0, 0, C);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int c = tile_row(m0, x), j = tile_col(n0, x);
                    hn[(size_t)c * DV + j0 + j] = fmaf(egc[c], S0T[j * P + c], au[x] - ae[x]);
                }
            }
            if (j0 + DB < DV) fetch_block(pf_s, hc, j0 + DB);
            __syncthreads();  // block's tiles consumed
        }
        }
    };
    for (int ci = 0; ci + 1 < n_chunks; ++ci) fwd_step(ci);  // every chunk before the last is full

    // ================= reverse sweep
    for (int ci = n_chunks - 1; ci >= 0; --ci) {
        const int t0 = ci * C;
        const int n = min(C, len - t0);
        __syncthreads();  // previous chunk done with every buffer; ds_run, h visible
        stage_a(t0, n, true);

        float* dG = scr;
        if constexpr (!MMA) {
        // ---------------- stage B: value-column blocks
        // dA entries (r2 + 16 (p >> 1), cl + 16 (p & 1)), p < 4, belong to task-1
        // thread t2: only it reads and writes them until the masking below
        if (task == 1) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int o = (r2 + 16 * (p >> 1)) * CP + cl + 16 * (p & 1);
                dAqk[o] = dAqb[o] = dAkk[o] = dAkb[o] = 0.f;
            }
        }
        float xq[NCI], xk[NCI], yk[NCI], yb[NCI];  // channel 4 cl + 64 g + e at [4 g + e]
#pragma unroll
        for (int i = 0; i < NCI; ++i) xq[i] = xk[i] = yk[i] = yb[i] = 0.f;
        float gcp = 0.f;                 // rowsum(dS_C * S0) of key channel tid (tid < DK)
        float dw_r0 = 0.f, dw_r1 = 0.f;  // scalar write gate: sums of v dU over value columns
        const float* hc = hbase + (size_t)ci * DK * DV;
        const float* dsc = ds_run + soff;
        float pf_s[NPF], pf_d[NPF];
        fetch_block(pf_s, hc, 0);
        fetch_block(pf_d, dsc, 0);

        for (int j0 = 0; j0 < DV; j0 += DB) {
            // B1: S0 and dS_C blocks (transposed), U, dO
            put_block(S0T, pf_s);
            put_block(dST, pf_d);
            {
                const int r = rr, j = cl;
                float u = 0.f, g = 0.f;
                if (r < n) {
                    const long long tok = tok_of(t0 + r), base = tok * DV;
                    u = gate_value(w, w_kind, tok, base, j0 + j) * to_f32(v[base + j0 + j]);
                    g = to_f32(dout[base + j0 + j]);
                }
                Ub[r * UP + j] = u;
                dOb[r * UP + j] = g;
            }
            __syncthreads();
            // B2: Y = Kh S0 + A_kk U (task 0);  dE = -A_qb^T dO - Bt dS_C (task 1)
            {
                const int j = cl, ra = r2, rb = r2 + 16;
                const float* X = task == 0 ? Kh : Bt;
                const float* ST = task == 0 ? S0T : dST;
                float o0 = 0.f, o1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll 4
                for (int c = 0; c < DK; c += 4) {
                    const float4 s4 = ld4(ST + j * P + c);
                    dot4_2(ld4(X + ra * P + c), s4, o0, p0);
                    dot4_2(ld4(X + rb * P + c), s4, o1, p1);
                }
                o0 += p0;
                o1 += p1;
                if (task == 0) {
                    for (int s = 0; s < ra; ++s) o0 = fmaf(Akk[ra * CP + s], Ub[s * UP + j], o0);
                    for (int s = 0; s < rb; ++s) o1 = fmaf(Akk[rb * CP + s], Ub[s * UP + j], o1);
                    Yb[ra * UP + j] = o0;
                    Yb[rb * UP + j] = o1;
                } else {
                    for (int s = ra; s < C; ++s) o0 = fmaf(Aqb[s * CP + ra], dOb[s * UP + j], o0);
                    for (int s = rb; s < C; ++s) o1 = fmaf(Aqb[s * CP + rb], dOb[s * UP + j], o1);
                    dEb[ra * UP + j] = -o0;
                    dEb[rb * UP + j] = -o1;
                }
            }
            __syncthreads();
            // B3: E = T Y (task 0);  dY = T^T dE (task 1)
            {
                const int j = cl, ra = r2, rb = r2 + 16;
                float o0 = 0.f, o1 = 0.f;
                if (task == 0) {
                    for (int s = 0; s <= ra; ++s) o0 = fmaf(Tm[ra * CP + s], Yb[s * UP + j], o0);
                    for (int s = 0; s <= rb; ++s) o1 = fmaf(Tm[rb * CP + s], Yb[s * UP + j], o1);
                    Eb[ra * UP + j] = o0;
                    Eb[rb * UP + j] = o1;
                } else {
                    for (int s = ra; s < C; ++s) o0 = fmaf(Tm[s * CP + ra], dEb[s * UP + j], o0);
                    for (int s = rb; s < C; ++s) o1 = fmaf(Tm[s * CP + rb], dEb[s * UP + j], o1);
                    dYb[ra * UP + j] = o0;
                    dYb[rb * UP + j] = o1;
                }
            }
            __syncthreads();
            // B4a: dU -> dv, dw (task 0);  dA (task 1)
            if (task == 0) {
                const int j = cl, ra = r2, rb = r2 + 16;
                float o0 = 0.f, o1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll 4
                for (int c = 0; c < DK; c += 4) {
                    const float4 d4 = ld4(dST + j * P + c);
                    dot4_2(ld4(Kt + ra * P + c), d4, o0, p0);
                    dot4_2(ld4(Kt + rb * P + c), d4, o1, p1);
                }
                o0 += p0;
                o1 += p1;
                for (int s = ra; s < C; ++s) o0 = fmaf(Aqk[s * CP + ra], dOb[s * UP + j], o0);
                for (int s = rb; s < C; ++s) o1 = fmaf(Aqk[s * CP + rb], dOb[s * UP + j], o1);
                for (int s = ra + 1; s < C; ++s) o0 = fmaf(Akk[s * CP + ra], dYb[s * UP + j], o0);
                for (int s = rb + 1; s < C; ++s) o1 = fmaf(Akk[s * CP + rb], dYb[s * UP + j], o1);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int r = h2 ? rb : ra;
                    const float du = h2 ? o1 : o0;
                    if (r < n) {
                        const long long tok = tok_of(t0 + r), base = tok * DV;
                        const float ww = gate_value(w, w_kind, tok, base, j0 + j);
                        const float vx = to_f32(v[base + j0 + j]);
                        dv[base + j0 + j] = from_f32<Tin>(ww * du);
                        if (w_kind == GDR_GATE_VECTOR) dw[base + j0 + j] = from_f32<Tin>(vx * du);
                        if (w_kind == GDR_GATE_FG2)  // through w = sqrt(beta^v)
                            dw[base + j0 + j] = from_f32<Tin>(vx * du / (2.f * ww));
                        if (h2) dw_r1 = fmaf(vx, du, dw_r1);
                        else dw_r0 = fmaf(vx, du, dw_r0);
                    }
                }
            } else {
                const int ra = r2, rb = r2 + 16, sa = cl, sb = cl + 16;
                float aqk[4], aqb[4], akk[4], akb[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int o = (r2 + 16 * (p >> 1)) * CP + cl + 16 * (p & 1);
                    aqk[p] = dAqk[o];
                    aqb[p] = dAqb[o];
                    akk[p] = dAkk[o];
                    akb[p] = dAkb[o];
                }
#pragma unroll
                for (int jj = 0; jj < DB; jj += 4) {
                    const float4 oa = ld4(dOb + ra * UP + jj), ob = ld4(dOb + rb * UP + jj);
                    const float4 ya = ld4(dYb + ra * UP + jj), yb4 = ld4(dYb + rb * UP + jj);
                    const float4 ua = ld4(Ub + sa * UP + jj), ub = ld4(Ub + sb * UP + jj);
                    const float4 ea = ld4(Eb + sa * UP + jj), eb = ld4(Eb + sb * UP + jj);
                    aqk[0] += dot4(oa, ua); aqk[1] += dot4(oa, ub);
                    aqk[2] += dot4(ob, ua); aqk[3] += dot4(ob, ub);
                    aqb[0] -= dot4(oa, ea); aqb[1] -= dot4(oa, eb);
                    aqb[2] -= dot4(ob, ea); aqb[3] -= dot4(ob, eb);
                    akk[0] += dot4(ya, ua); akk[1] += dot4(ya, ub);
                    akk[2] += dot4(yb4, ua); akk[3] += dot4(yb4, ub);
                    akb[0] -= dot4(ya, ea); akb[1] -= dot4(ya, eb);
                    akb[2] -= dot4(yb4, ea); akb[3] -= dot4(yb4, eb);
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int o = (r2 + 16 * (p >> 1)) * CP + cl + 16 * (p & 1);
                    dAqk[o] = aqk[p];
                    dAqb[o] = aqb[p];
                    dAkk[o] = akk[p];
                    dAkb[o] = akb[p];
                }
            }
            // B4b: the [C][DK] sums, the dG_C share, and dS0 of this block
#pragma unroll
            for (int jj = 0; jj < DB; jj += 4) {
                const float4 o4 = ld4(dOb + rr * UP + jj), y4 = ld4(dYb + rr * UP + jj);
                const float4 u4 = ld4(Ub + rr * UP + jj), e4 = ld4(Eb + rr * UP + jj);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = jj + e;
                    const float go = comp(o4, e), gy = comp(y4, e), gu = comp(u4, e), ge = comp(e4, e);
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        const int c = 4 * cl + 64 * g;
                        const float4 s4 = ld4(S0T + j * P + c), d4 = ld4(dST + j * P + c);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            xq[4 * g + x] = fmaf(go, comp(s4, x), xq[4 * g + x]);
                            xk[4 * g + x] = fmaf(gy, comp(s4, x), xk[4 * g + x]);
                            yk[4 * g + x] = fmaf(gu, comp(d4, x), yk[4 * g + x]);
                            yb[4 * g + x] = fmaf(-ge, comp(d4, x), yb[4 * g + x]);
                        }
                    }
                }
            }
            if (tid < DK) {
#pragma unroll 4
                for (int j = 0; j < DB; ++j) gcp = fmaf(dST[j * P + tid], S0T[j * P + tid], gcp);
            }
            if (rr < DK / 4) {  // dS0 = e^G_C dS_C + Qh^T dO + Kh^T dY, channels 4 rr ..
                const int c = 4 * rr, j = cl;
                const float4 g4 = ld4(egc + c), d4 = ld4(dST + j * P + c);
                float acc[4] = {g4.x * d4.x, g4.y * d4.y, g4.z * d4.z, g4.w * d4.w};
#pragma unroll 4
                for (int r = 0; r < n; ++r) {
                    const float4 qh = ld4(Qh + r * P + c), kh = ld4(Kh + r * P + c);
                    const float go = dOb[r * UP + j], gy = dYb[r * UP + j];
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        acc[x] = fmaf(comp(qh, x), go, fmaf(comp(kh, x), gy, acc[x]));
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) ds_run[soff + (size_t)(c + x) * DV + j0 + j] = acc[x];
            }
            if (j0 + DB < DV) {  // next block's columns: not written by this chunk yet
                fetch_block(pf_s, hc, j0 + DB);
                fetch_block(pf_d, dsc, j0 + DB);
            }
            __syncthreads();  // block's tiles consumed before the next block loads
        }

        // scalar write gate: one value per token (task-0 warps hold the row sums)
        if (w_kind == GDR_GATE_SCALAR && task == 0) {
#pragma unroll
            for (int m = 8; m >= 1; m >>= 1) {
                dw_r0 += __shfl_xor_sync(0xffffffffu, dw_r0, m);
                dw_r1 += __shfl_xor_sync(0xffffffffu, dw_r1, m);
            }
            if (cl == 0 && r2 < n) dw[tok_of(t0 + r2)] = from_f32<Tin>(dw_r0);
            if (cl == 0 && r2 + 16 < n) dw[tok_of(t0 + r2 + 16)] = from_f32<Tin>(dw_r1);
        }

        // gradient on G_C: e^G_C rowsum(dS_C S0) + colsum(Kt YK + Bt YB), taken
        // before the grams' shares join YK and YB (rows summed in a fixed order)
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int c = 4 * cl + 64 * g;
            const float4 kt = ld4(Kt + rr * P + c), bt = ld4(Bt + rr * P + c);
            store4(gcr + rr * P + c, kt.x * yk[4 * g] + bt.x * yb[4 * g],
                   kt.y * yk[4 * g + 1] + bt.y * yb[4 * g + 1],
                   kt.z * yk[4 * g + 2] + bt.z * yb[4 * g + 2],
                   kt.w * yk[4 * g + 3] + bt.w * yb[4 * g + 3]);
        }
        // dA masks (their owners, as above)
        if (task == 1) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int r = r2 + 16 * (p >> 1), s = cl + 16 * (p & 1);
                if (s > r) dAqk[r * CP + s] = dAqb[r * CP + s] = 0.f;
                if (s >= r) dAkk[r * CP + s] = dAkb[r * CP + s] = 0.f;
            }
        }
        __syncthreads();
        if (tid < DK) {
            float g = egc[tid] * gcp;
            for (int r = 0; r < C; ++r) g += gcr[r * P + tid];
            dgc[tid] = g;
        }

        // ---------------- stage C: the grams' gradients (e^-G_C folded into the operands)
        {
            const int r = rr;
            float4 ig[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) ig[g] = ld4(igc + 4 * cl + 64 * g);
            for (int s = 0; s < C; ++s) {
                const float gqk = dAqk[r * CP + s], gqb = dAqb[r * CP + s];
                const float gkk = dAkk[r * CP + s], gkb = dAkb[r * CP + s];
                const float tqk = dAqk[s * CP + r], tqb = dAqb[s * CP + r];
                const float tkk = dAkk[s * CP + r], tkb = dAkb[s * CP + r];
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const int c = 4 * cl + 64 * g;
                    const float4 kt = ld4(Kt + s * P + c), bt = ld4(Bt + s * P + c);
                    const float4 qh = ld4(Qh + s * P + c), kh = ld4(Kh + s * P + c);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float f = comp(ig[g], x);
                        const float ktf = comp(kt, x) * f, btf = comp(bt, x) * f;
                        const float qhf = comp(qh, x) * f, khf = comp(kh, x) * f;
                        const int i = 4 * g + x;
                        xq[i] = fmaf(gqk, ktf, fmaf(gqb, btf, xq[i]));
                        xk[i] = fmaf(gkk, ktf, fmaf(gkb, btf, xk[i]));
                        yk[i] = fmaf(tqk, qhf, fmaf(tkk, khf, yk[i]));
                        yb[i] = fmaf(tqb, qhf, fmaf(tkb, khf, yb[i]));
                    }
                }
            }
        }
        __syncthreads();  // dA reads done: the scratch becomes dG

        // ---------------- stage D: back to q, k, b and the decay
        {
            const int r = rr;
            float db_row = 0.f;
            const long long tok = tok_of(t0 + min(r, n - 1)), base = tok * DK;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int c = 4 * cl + 64 * g;
                float gq[4], gk[4], gb[4], gg[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int i = 4 * g + x;
                    const float gr = Gs[r * P + c + x], gc = Gs[(C - 1) * P + c + x];
                    const float eg = __expf(gr), et = __expf(gc - gr);
                    const float kt = Kt[r * P + c + x], bt = Bt[r * P + c + x];
                    gq[x] = eg * xq[i];
                    const float bg = fg2_b ? 1.f : Bs[r * P + c + x];
                    gk[x] = fmaf(eg, xk[i], et * (yk[i] + bg * yb[i]));
                    gb[x] = kt * yb[i];
                    if (fg2_b) {  // through k~ = sqrt(beta^k) k
                        const float sb = Bs[r * P + c + x];
                        gb[x] = gk[x] * to_f32(k[base + c + x]) / (2.f * sb);
                        gk[x] *= sb;
                    }
                    db_row += gb[x];
                    gg[x] = Qh[r * P + c + x] * xq[i] + Kh[r * P + c + x] * xk[i] - kt * yk[i] -
                            bt * yb[i];
                    if (r == n - 1) gg[x] += dgc[c + x];
                    if (r >= n) gg[x] = 0.f;
                }
                store4(dG + r * P + c, gg[0], gg[1], gg[2], gg[3]);
                if (r < n) {
                    store4(dq + base + c, gq[0], gq[1], gq[2], gq[3]);
                    store4(dk + base + c, gk[0], gk[1], gk[2], gk[3]);
                    if (b_kind == GDR_GATE_VECTOR || fg2_b)
                        store4(db + base + c, gb[0], gb[1], gb[2], gb[3]);
                }
            }
            if (b_kind == GDR_GATE_SCALAR) {
#pragma unroll
                for (int m = 8; m >= 1; m >>= 1) db_row += __shfl_xor_sync(0xffffffffu, db_row, m);
                if (cl == 0 && r < n) db[tok_of(t0 + r)] = from_f32<Tin>(db_row);
            }
        }
        } else {
        // ---------------- stages B-D on the tensor cores
        {
            const int wid = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
            constexpr int NTN = DK / 8;   // 8-wide column tiles across DK
            constexpr int NTW = DK / 64;  // [C][DK] tiles per warp, of each of the four sums
            float xq[NTW][4], xk[NTW][4], yk[NTW][4], yb[NTW][4];  // yb holds +E dS^T until negated
            float dacc[2][4];  // this warp's dA tiles: ids 2 wid, 2 wid + 1 (matrix id >> 3)
#pragma unroll
            for (int u = 0; u < NTW; ++u)
#pragma unroll
                for (int x = 0; x < 4; ++x) xq[u][x] = xk[u][x] = yk[u][x] = yb[u][x] = 0.f;
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int x = 0; x < 4; ++x) dacc[u][x] = 0.f;
            if (tid < 2 * C) dwp[tid] = 0.f;
            float gcp = 0.f;  // rowsum(dS_C * S0) of key channel tid (tid < DK)
            const float* hc = hbase + (size_t)ci * DK * DV;
            const float* dsc = ds_run + soff;
            float pf_s[NPF], pf_d[NPF];
            fetch_block(pf_s, hc, 0);
            fetch_block(pf_d, dsc, 0);

            for (int j0 = 0; j0 < DV; j0 += DB) {
                put_block(S0T, pf_s);
                put_block(dST, pf_d);
                {
                    const int r = rr, j = cl;
                    float u = 0.f, gg = 0.f;
                    if (r < n) {
                        const long long tok = tok_of(t0 + r), base = tok * DV;
                        u = gate_value(w, w_kind, tok, base, j0 + j) * to_f32(v[base + j0 + j]);
                        gg = to_f32(dout[base + j0 + j]);
                    }
                    Ub[r * UP + j] = u;
                    dOb[r * UP + j] = gg;
                }
                __syncthreads();
                // B2: Y = Kh S0 + A_kk U (warps 0-3);  dE = -(Bt dS_C + A_qb^T dO) (warps 4-7)
                if (wid < 8) {
                    const int q4 = wid & 3, m0 = 16 * (q4 >> 1), n0 = 8 * (q4 & 1);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    if (wid < 4) {
                        mma_tile<false, false>(acc, Kh, P, S0T, P, m0, n0, 0, DK);
                        mma_tile<false, true>(acc, Akk, CP, Ub, UP, m0, n0, 0, C);
                        store_tile(Yb, UP, m0, n0, acc);
                    } else {
                        mma_tile<false, false>(acc, Bt, P, dST, P, m0, n0, 0, DK);
                        mma_tile<true, true>(acc, Aqb, CP, dOb, UP, m0, n0, 0, C);
                        store_tile(dEb, UP, m0, n0, acc, -1.f);
                    }
                }
                __syncthreads();
                // B3: E = T Y (warps 0-3);  dY = T^T dE (warps 4-7)
                if (wid < 8) {
                    const int q4 = wid & 3, m0 = 16 * (q4 >> 1), n0 = 8 * (q4 & 1);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    if (wid < 4) {
                        mma_tile<false, true>(acc, Tm, CP, Yb, UP, m0, n0, 0, C);
                        store_tile(Eb, UP, m0, n0, acc);
                    } else {
                        mma_tile<true, true>(acc, Tm, CP, dEb, UP, m0, n0, 0, C);
                        store_tile(dYb, UP, m0, n0, acc);
                    }
                }
                __syncthreads();
                // B4a: dU -> dv, dw (warps 0-3)
                if (wid < 4) {
                    const int m0 = 16 * (wid >> 1), n0 = 8 * (wid & 1);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_tile<false, false>(acc, Kt, P, dST, P, m0, n0, 0, DK);
                    mma_tile<true, true>(acc, Aqk, CP, dOb, UP, m0, n0, 0, C);
                    mma_tile<true, true>(acc, Akk, CP, dYb, UP, m0, n0, 0, C);
                    float rs[2] = {0.f, 0.f};  // v dU over this tile's columns, rows m0 + g (+ 8)
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int r = tile_row(m0, x), j = tile_col(n0, x);
                        if (r < n) {
                            const long long tok = tok_of(t0 + r), base = tok * DV;
                            const float ww = gate_value(w, w_kind, tok, base, j0 + j);
                            const float vx = to_f32(v[base + j0 + j]);
                            dv[base + j0 + j] = from_f32<Tin>(ww * acc[x]);
                            if (w_kind == GDR_GATE_VECTOR) dw[base + j0 + j] = from_f32<Tin>(vx * acc[x]);
                            if (w_kind == GDR_GATE_FG2)  // through w = sqrt(beta^v)
                                dw[base + j0 + j] = from_f32<Tin>(vx * acc[x] / (2.f * ww));
                            rs[x >> 1] = fmaf(vx, acc[x], rs[x >> 1]);
                        }
                    }
                    if (w_kind == GDR_GATE_SCALAR) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
                            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
                        }
                        if (t == 0) {  // this warp alone owns these entries
                            dwp[(wid & 1) * C + m0 + g] += rs[0];
                            dwp[(wid & 1) * C + m0 + g + 8] += rs[1];
                        }
                    }
                }
                // dA: dO U^T, dO E^T, dY U^T, dY E^T (the E ones negated at the masking)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int id = 2 * wid + u, mat = id >> 3, rem = id & 7;
                    const int m0 = 16 * (rem >> 2), n0 = 8 * (rem & 3);
                    mma_tile<false, false>(dacc[u], (mat & 2) ? dYb : dOb, UP, (mat & 1) ? Eb : Ub,
                                           UP, m0, n0, 0, DB);
                }
                // B4b: XQ += dO S0^T, XK += dY S0^T, YK += U dS_C^T, YB += E dS_C^T
#pragma unroll
                for (int u = 0; u < NTW; ++u) {
                    const int id = NTW * wid + u, m0 = 16 * (id / NTN), n0 = 8 * (id % NTN);
                    mma_tile<false, true>(xq[u], dOb, UP, S0T, P, m0, n0, 0, DB);
                    mma_tile<false, true>(xk[u], dYb, UP, S0T, P, m0, n0, 0, DB);
                    mma_tile<false, true>(yk[u], Ub, UP, dST, P, m0, n0, 0, DB);
                    mma_tile<false, true>(yb[u], Eb, UP, dST, P, m0, n0, 0, DB);
                }
                if (tid < DK) {
#pragma unroll 4
                    for (int j = 0; j < DB; ++j) gcp = fmaf(dST[j * P + tid], S0T[j * P + tid], gcp);
                }
                if (wid < DK / 8) {  // dS0 = e^G_C dS_C + Qh^T dO + Kh^T dY
                    const int m0 = 16 * (wid >> 1), n0 = 8 * (wid & 1);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_tile<true, true>(acc, Qh, P, dOb, UP, m0, n0, 0, C);
                    mma_tile<true, true>(acc, Kh, P, dYb, UP, m0, n0, 0, C);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int c = tile_row(m0, x), j = tile_col(n0, x);
                        ds_run[soff + (size_t)c * DV + j0 + j] = fmaf(egc[c], dST[j * P + c], acc[x]);
                    }
                }
                if (j0 + DB < DV) {  // next block's columns: not written by this chunk yet
                    fetch_block(pf_s, hc, j0 + DB);
                    fetch_block(pf_d, dsc, j0 + DB);
                }
                __syncthreads();  // block's tiles consumed before the next block loads
            }

            // scalar write gate: one value per token
            if (w_kind == GDR_GATE_SCALAR && tid < n)
                dw[tok_of(t0 + tid)] = from_f32<Tin>(dwp[tid] + dwp[C + tid]);

            // YB's stage-B share is -E dS_C^T; gradient on G_C: e^G_C rowsum(dS_C S0) +
            // colsum(Kt YK + Bt YB) before the grams' shares join, per row half in gcr
#pragma unroll
            for (int u = 0; u < NTW; ++u) {
                const int id = NTW * wid + u, mt = id / NTN, m0 = 16 * mt, n0 = 8 * (id % NTN);
                float cs[2] = {0.f, 0.f};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    yb[u][x] = -yb[u][x];
                    const int r = tile_row(m0, x), c = tile_col(n0, x);
                    cs[x & 1] += Kt[r * P + c] * yk[u][x] + Bt[r * P + c] * yb[u][x];
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    cs[h] += __shfl_xor_sync(0xffffffffu, cs[h], 4);
                    cs[h] += __shfl_xor_sync(0xffffffffu, cs[h], 8);
                    cs[h] += __shfl_xor_sync(0xffffffffu, cs[h], 16);
                }
                if (g == 0) {
                    gcr[mt * P + n0 + 2 * t] = cs[0];
                    gcr[mt * P + n0 + 2 * t + 1] = cs[1];
                }
            }
            // masked dA into shared memory
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int id = 2 * wid + u, mat = id >> 3, rem = id & 7;
                const int m0 = 16 * (rem >> 2), n0 = 8 * (rem & 3);
                float* dst = dAqk + mat * C * CP;
                const float sgn = (mat & 1) ? -1.f : 1.f;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int r = tile_row(m0, x), sc = tile_col(n0, x);
                    const bool keep = (mat >= 2) ? (sc < r) : (sc <= r);
                    dst[r * CP + sc] = keep ? sgn * dacc[u][x] : 0.f;
                }
            }
            __syncthreads();
            if (tid < DK) dgc[tid] = egc[tid] * gcp + gcr[tid] + gcr[P + tid];

            // ---------------- stage C: the grams' gradients, e^-G_C per key channel
#pragma unroll
            for (int u = 0; u < NTW; ++u) {
                const int id = NTW * wid + u, m0 = 16 * (id / NTN), n0 = 8 * (id % NTN);
                float tq[4] = {0.f, 0.f, 0.f, 0.f}, tk[4] = {0.f, 0.f, 0.f, 0.f};
                float ty[4] = {0.f, 0.f, 0.f, 0.f}, tb[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tile<false, true>(tq, dAqk, CP, Kt, P, m0, n0, 0, C);
                mma_tile<false, true>(tq, dAqb, CP, Bt, P, m0, n0, 0, C);
                mma_tile<false, true>(tk, dAkk, CP, Kt, P, m0, n0, 0, C);
                mma_tile<false, true>(tk, dAkb, CP, Bt, P, m0, n0, 0, C);
                mma_tile<true, true>(ty, dAqk, CP, Qh, P, m0, n0, 0, C);
                mma_tile<true, true>(ty, dAkk, CP, Kh, P, m0, n0, 0, C);
                mma_tile<true, true>(tb, dAqb, CP, Qh, P, m0, n0, 0, C);
                mma_tile<true, true>(tb, dAkb, CP, Kh, P, m0, n0, 0, C);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float f = igc[tile_col(n0, x)];
                    xq[u][x] = fmaf(f, tq[x], xq[u][x]);
                    xk[u][x] = fmaf(f, tk[x], xk[u][x]);
                    yk[u][x] = fmaf(f, ty[x], yk[u][x]);
                    yb[u][x] = fmaf(f, tb[x], yb[u][x]);
                }
            }
            __syncthreads();  // dA and gcr reads done: the scratch becomes dG, gcr the db rows

            // ---------------- stage D: back to q, k, b and the decay
#pragma unroll
            for (int u = 0; u < NTW; ++u) {
                const int id = NTW * wid + u, m0 = 16 * (id / NTN), n0 = 8 * (id % NTN);
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // rows m0 + g + 8 h, columns c0, c0 + 1
                    const int r = m0 + g + 8 * h, c0 = n0 + 2 * t;
                    float gq[2], gk[2], gb[2], gg[2];
                    const long long tok = tok_of(t0 + min(r, n - 1)), base = tok * DK;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int x = 2 * h + e, c = c0 + e;
                        const float gr = Gs[r * P + c], gc = Gs[(C - 1) * P + c];
                        const float eg = __expf(gr), et = __expf(gc - gr);
                        const float kt = Kt[r * P + c], bt = Bt[r * P + c];
                        const float bgate = fg2_b ? 1.f : Bs[r * P + c];
                        gq[e] = eg * xq[u][x];
                        gk[e] = fmaf(eg, xk[u][x], et * (yk[u][x] + bgate * yb[u][x]));
                        gb[e] = kt * yb[u][x];
                        if (fg2_b) {  // through k~ = sqrt(beta^k) k
                            const float sb = Bs[r * P + c];
                            gb[e] = gk[e] * to_f32(k[base + c]) / (2.f * sb);
                            gk[e] *= sb;
                        }
                        gg[e] = Qh[r * P + c] * xq[u][x] + Kh[r * P + c] * xk[u][x] -
                                kt * yk[u][x] - bt * yb[u][x];
                        if (r == n - 1) gg[e] += dgc[c];
                        if (r >= n) gg[e] = 0.f;
                        gcr[r * P + c] = r < n ? gb[e] : 0.f;
                    }
                    store2(dG + r * P + c0, gg[0], gg[1]);
                    if (r < n) {
                        store2(dq + base + c0, gq[0], gq[1]);
                        store2(dk + base + c0, gk[0], gk[1]);
                        if (b_kind == GDR_GATE_VECTOR || fg2_b) store2(db + base + c0, gb[0], gb[1]);
                    }
                }
            }
            if (b_kind == GDR_GATE_SCALAR) {
                __syncthreads();
                if (tid < n) {
                    float sum = 0.f;
                    for (int c = 0; c < DK; ++c) sum += gcr[tid * P + c];
                    db[tok_of(t0 + tid)] = from_f32<Tin>(sum);
                }
            }
        }
        }
        __syncthreads();
        if (a_kind != GDR_GATE_ONE) {
            if (tid < DK) {  // d log a_r = sum_{r' >= r} dG_r';  da = d log a / a
                const int c = tid;
                float run = 0.f;
                for (int r = n - 1; r >= 0; --r) {
                    run += dG[r * P + c];
                    const float g = run / As[r * P + c];
                    if (a_kind == GDR_GATE_VECTOR) da[(tok_of(t0 + r)) * DK + c] = from_f32<Tin>(g);
                    else dG[r * P + c] = g;
                }
            }
            if (a_kind == GDR_GATE_SCALAR) {
                __syncthreads();
                float s = 0.f;
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const float4 d4 = ld4(dG + rr * P + 4 * cl + 64 * g);
                    s += d4.x + d4.y + d4.z + d4.w;
                }
#pragma unroll
                for (int m = 8; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
                if (cl == 0 && rr < n) da[tok_of(t0 + rr)] = from_f32<Tin>(s);
            }
        }
    }
    __syncthreads();
    if (ds0) {
        for (int x = tid; x < DK * DV; x += NT) ds0[soff + x] = ds_run[soff + x];
    }
}

template <typename Tin, int DK, int DV>
static cudaError_t launch_backward_t(const gdr_desc& d, const int* cu_seqlens, int n_seqs,
                                     const void* const* in, const float* s0,
                                     const void* dout, const float* ds_final, float* hs,
                                     float* ds_run, void* const* grads, float* ds0,
                                     int* err_word, cudaStream_t st) {
    auto kern = backward_kernel<Tin, DK, DV, sizeof(Tin) == 2>;  // bf16: tensor cores
    const size_t smem = BwdSmem<DK>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const long long nseq = cu_seqlens ? n_seqs : d.B;
    kern<<<(unsigned)(nseq * d.H), BW_NT, smem, st>>>(
        d.T, d.H, cu_seqlens, (const Tin*)in[0], (const Tin*)in[1], (const Tin*)in[2], (const Tin*)in[3],
        (const Tin*)in[4], (const Tin*)in[5], (int)d.decay, (int)d.erase, (int)d.write,
        (const Tin*)dout, s0, ds_final, hs, ds_run, (Tin*)grads[0], (Tin*)grads[1],
        (Tin*)grads[2], (Tin*)grads[3], (Tin*)grads[4], (Tin*)grads[5], ds0, err_word);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_backward_d(const gdr_desc& d, const int* cu_seqlens, int n_seqs,
                                     const void* const* in, const float* s0,
                                     const void* dout, const float* ds_final, float* hs,
                                     float* ds_run, void* const* grads, float* ds0,
                                     int* err_word, cudaStream_t st) {
#define GDR_BWD(DK_, DV_)                                                                  \
    if (d.dk == DK_ && d.dv == DV_)                                                        \
        return launch_backward_t<Tin, DK_, DV_>(d, cu_seqlens, n_seqs, in, s0, dout, ds_final, \
                                                hs, ds_run, grads, ds0, err_word, st);
    GDR_BWD(128, 128)
    GDR_BWD(128, 64)
    GDR_BWD(64, 128)
    GDR_BWD(64, 64)
#undef GDR_BWD
    return cudaErrorInvalidValue;
}

// Chunk-start states: B sequences of ceil(T / 32) chunks each, or packed
// sequences with at most ceil(T / 32) + n_seqs chunks in all (their lengths
// sum to at most T), for each of the H heads.
static size_t state_matrices(const gdr_desc& d, bool packed, int n_seqs) {
    const size_t nc = ((size_t)d.T + BW_C - 1) / BW_C;
    return packed ? (nc + (size_t)n_seqs) * d.H : nc * d.B * d.H;
}

bool backward_tc_supports(const gdr_desc& d, bool packed);
size_t backward_tc_workspace_bytes(const gdr_desc& d);
cudaError_t launch_backward_tc(const gdr_desc& d, const void* const* in, const float* s0,
                               const void* dout, const float* ds_final, void* const* grads,
                               float* ds0, void* workspace, int* err_word, cudaStream_t st);

// n_seqs > 0: packed sequences; 0: the B batch rows.
size_t backward_workspace_bytes(const gdr_desc& d, int n_seqs) {
    if (backward_tc_supports(d, n_seqs > 0)) return backward_tc_workspace_bytes(d);
    const size_t mat = (size_t)d.dk * d.dv * sizeof(float);
    const size_t nseq = n_seqs > 0 ? (size_t)n_seqs : (size_t)d.B;
    // chunk-start states, then the running dS of every (sequence, head)
    return mat * (state_matrices(d, n_seqs > 0, n_seqs) + nseq * d.H);
}

// in = {q, k, v, a, b, w}; grads = {dq, dk, dv, da, db, dw}.  bf16 with
// dk = dv = 128 and one sequence per batch row runs on the tensor cores
// (bwd_tc.cu); everything else on this file's kernel.
cudaError_t launch_backward(const gdr_desc& d, const int* cu_seqlens, int n_seqs,
                            const void* const* in, const float* s0, const void* dout,
                            const float* ds_final, void* const* grads, float* ds0,
                            void* workspace, int* err_word, cudaStream_t st) {
    if (backward_tc_supports(d, cu_seqlens != nullptr))
        return launch_backward_tc(d, in, s0, dout, ds_final, grads, ds0, workspace, err_word, st);
    float* hs = static_cast<float*>(workspace);
    float* ds_run = hs + state_matrices(d, cu_seqlens != nullptr, n_seqs) * d.dk * d.dv;
    if (d.in_dtype == GDR_BF16)
        return launch_backward_d<__nv_bfloat16>(d, cu_seqlens, n_seqs, in, s0, dout, ds_final,
                                                hs, ds_run, grads, ds0, err_word, st);
    return launch_backward_d<float>(d, cu_seqlens, n_seqs, in, s0, dout, ds_final, hs, ds_run,
                                    grads, ds0, err_word, st);
}

}  // namespace gdr
