// backward.cu -- gradients of the chunked gated delta rule, float32 on the
// CUDA cores.
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
// Two launches.  The float32 forward kernel (chunk 32) stores the state at the
// start of every chunk in the workspace.  This kernel then takes one
// (batch, head) per CTA and walks the chunks backwards, carrying dS in the
// workspace (L2-resident, one [dk, dv] matrix per head).  Per chunk: stage A
// forms the gated operands, the four grams and T; stage B runs the dv-side
// products in blocks of 16 value columns, keeping dA and the C x dk gradient
// sums in registers; stage C adds the grams' gradients; stage D maps the
// sums back to q, k, b and the decay.
#include "common.cuh"

namespace gdr {

constexpr int BW_C = 32;    // tokens per chunk
constexpr int BW_DB = 16;   // value columns per stage-B block
constexpr int BW_NT = 512;  // threads: one per (row, column) of a [C][DB] tile
constexpr float BW_MIN_LOG_DECAY = -80.0f;

template <int DK>
struct BwdSmem {
    static constexpr int C = BW_C, DB = BW_DB;
    static constexpr int P = DK + 1;   // row stride of [C][DK] tiles
    static constexpr int CP = C + 1;   // row stride of [C][C] tiles
    static constexpr int SP = DB + 1;  // row stride of [DK][DB] and [C][DB] tiles
    static constexpr int kQh = 0;
    static constexpr int kKh = kQh + C * P;
    static constexpr int kKt = kKh + C * P;
    static constexpr int kBt = kKt + C * P;
    static constexpr int kB = kBt + C * P;  // erase gate
    static constexpr int kG = kB + C * P;   // cumulative log decay
    static constexpr int kAqk = kG + C * P;
    static constexpr int kAqb = kAqk + C * CP;
    static constexpr int kAkk = kAqb + C * CP;
    static constexpr int kAkb = kAkk + C * CP;
    static constexpr int kT = kAkb + C * CP;
    static constexpr int kScr = kT + C * CP;
    // stage B tiles inside the scratch
    static constexpr int sS0 = 0;
    static constexpr int sdS = sS0 + DK * SP;
    static constexpr int sU = sdS + DK * SP;
    static constexpr int sdO = sU + C * SP;
    static constexpr int sY = sdO + C * SP;
    static constexpr int sE = sY + C * SP;
    static constexpr int sdE = sE + C * SP;
    static constexpr int sdY = sdE + C * SP;
    static constexpr int scrB = sdY + C * SP;
    // stage C: masked dA_qk, dA_qb, dA_kk, dA_kb; stage D: dG [C][P]
    static constexpr int scrC = 4 * C * CP;
    static constexpr int scrD = C * P;
    static constexpr int scr = scrB > scrC ? (scrB > scrD ? scrB : scrD) : (scrC > scrD ? scrC : scrD);
    static constexpr int kGcr = kScr + scr;  // per-row shares of the G_C gradient [C][P]
    static constexpr int kEgc = kGcr + C * P;  // e^G_C per channel
    static constexpr int kIgc = kEgc + DK;   // e^-G_C
    static constexpr int kDgc = kIgc + DK;   // gradient on G_C
    static constexpr int floats = kDgc + DK;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(BW_NT, 1)
backward_kernel(int T, int H, const Tin* __restrict__ q, const Tin* __restrict__ k,
                const Tin* __restrict__ v, const Tin* __restrict__ a,
                const Tin* __restrict__ b, const Tin* __restrict__ w, int a_kind, int b_kind,
                int w_kind, const Tin* __restrict__ dout, const float* __restrict__ ds_final,
                const float* __restrict__ hs, float* __restrict__ ds_run,
                Tin* __restrict__ dq, Tin* __restrict__ dk, Tin* __restrict__ dv,
                Tin* __restrict__ da, Tin* __restrict__ db, Tin* __restrict__ dw,
                float* __restrict__ ds0, int* __restrict__ err_word) {
    using L = BwdSmem<DK>;
    constexpr int C = BW_C, DB = BW_DB, NT = BW_NT;
    constexpr int P = L::P, CP = L::CP, SP = L::SP;
    constexpr int NCI = DK / 16;  // key channels per thread in the [C][DK] sums
    static_assert(C * DB == NT && DV % DB == 0 && DK % 16 == 0, "shape");

    extern __shared__ float sm[];
    float* Qh = sm + L::kQh;
    float* Kh = sm + L::kKh;
    float* Kt = sm + L::kKt;
    float* Bt = sm + L::kBt;
    float* Bs = sm + L::kB;
    float* Gs = sm + L::kG;
    float* Aqk = sm + L::kAqk;
    float* Aqb = sm + L::kAqb;
    float* Akk = sm + L::kAkk;
    float* Akb = sm + L::kAkb;
    float* Tm = sm + L::kT;
    float* scr = sm + L::kScr;
    float* S0b = scr + L::sS0;
    float* dSb = scr + L::sdS;
    float* Ub = scr + L::sU;
    float* dOb = scr + L::sdO;
    float* Yb = scr + L::sY;
    float* Eb = scr + L::sE;
    float* dEb = scr + L::sdE;
    float* dYb = scr + L::sdY;
    float* egc = sm + L::kEgc;
    float* igc = sm + L::kIgc;
    float* dgc = sm + L::kDgc;
    float* gcr = sm + L::kGcr;

    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int bi = bh / H, hi = bh % H;
    const int rr = tid >> 4;  // row of this thread in [C][*] tiles
    const int cl = tid & 15;  // column lane: value column in stage B, key channels cl + 16 i
    const int n_chunks = (T + C - 1) / C;
    const size_t soff = (size_t)bh * DK * DV;
    auto tok_of = [&](int t) { return ((long long)bi * T + t) * H + hi; };

    for (int x = tid; x < DK * DV; x += NT) ds_run[soff + x] = ds_final ? ds_final[soff + x] : 0.f;

    for (int ci = n_chunks - 1; ci >= 0; --ci) {
        const int t0 = ci * C;
        const int n = min(C, T - t0);
        __syncthreads();  // previous chunk done with every buffer; ds_run visible

        // ---------------- stage A: gated operands, grams, T
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f;
            if (r < n) {
                const long long tok = tok_of(t0 + r), base = tok * DK;
                qv = to_f32(q[base + c]);
                kv = to_f32(k[base + c]);
                bv = gate_value(b, b_kind, tok, base, c);
                gv = a_kind == GDR_GATE_ONE ? 0.f
                                            : safe_log_decay(gate_value(a, a_kind, tok, base, c));
            }
            Qh[r * P + c] = qv;
            Kh[r * P + c] = kv;
            Bs[r * P + c] = bv;
            Gs[r * P + c] = gv;
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
            Bt[r * P + c] = Bs[r * P + c] * kv * et;
        }
        __syncthreads();
        {
            const int r = rr;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int s = cl + 16 * h2;
                float qk = 0.f, qb = 0.f, kk = 0.f, kb = 0.f;
                if (s <= r) {
#pragma unroll 4
                    for (int c = 0; c < DK; ++c) {
                        const float kbs = Kt[s * P + c] * igc[c];
                        const float bbs = Bt[s * P + c] * igc[c];
                        const float qr = Qh[r * P + c], kr = Kh[r * P + c];
                        qk = fmaf(qr, kbs, qk);
                        qb = fmaf(qr, bbs, qb);
                        kk = fmaf(kr, kbs, kk);
                        kb = fmaf(kr, bbs, kb);
                    }
                }
                Aqk[r * CP + s] = qk;
                Aqb[r * CP + s] = qb;
                Akk[r * CP + s] = s < r ? kk : 0.f;
                Akb[r * CP + s] = s < r ? kb : 0.f;
            }
        }
        __syncthreads();
        if (tid < C) {  // column j = tid of T = (I + A_kb)^-1, forward substitution
            const int j = tid;
            for (int i = 0; i < C; ++i) {
                float t = (i == j) ? 1.f : 0.f;
                if (i > j) {
                    for (int s = j; s < i; ++s) t = fmaf(-Akb[i * CP + s], Tm[s * CP + j], t);
                }
                Tm[i * CP + j] = t;
            }
        }
        __syncthreads();

        // ---------------- stage B: value-column blocks
        float aqk[2] = {0.f, 0.f}, aqb[2] = {0.f, 0.f}, akk[2] = {0.f, 0.f}, akb[2] = {0.f, 0.f};
        float xq[NCI], xk[NCI], yk[NCI], yb[NCI];
#pragma unroll
        for (int i = 0; i < NCI; ++i) xq[i] = xk[i] = yk[i] = yb[i] = 0.f;
        float gcp = 0.f;    // rowsum(dS_C * S0) of key channel tid (tid < DK)
        float dw_row = 0.f; // scalar write gate: sum over value columns of v dU
        const float* hc = hs + ((size_t)bh * n_chunks + ci) * DK * DV;

        for (int j0 = 0; j0 < DV; j0 += DB) {
            // B1: load S0, dS_C, U, dO blocks
            for (int x = tid; x < DK * DB; x += NT) {
                const int c = x / DB, j = x % DB;
                S0b[c * SP + j] = hc[(size_t)c * DV + j0 + j];
                dSb[c * SP + j] = ds_run[soff + (size_t)c * DV + j0 + j];
            }
            float wv = 0.f, vv = 0.f;
            {
                const int r = rr, j = cl;
                float u = 0.f, g = 0.f;
                if (r < n) {
                    const long long tok = tok_of(t0 + r), base = tok * DV;
                    vv = to_f32(v[base + j0 + j]);
                    wv = gate_value(w, w_kind, tok, base, j0 + j);
                    u = wv * vv;
                    g = to_f32(dout[base + j0 + j]);
                }
                Ub[r * SP + j] = u;
                dOb[r * SP + j] = g;
            }
            __syncthreads();
            // B2: Y = Kh S0 + A_kk U;  dE = -A_qb^T dO - Bt dS_C
            {
                const int r = rr, j = cl;
                float y = 0.f, de = 0.f;
#pragma unroll 4
                for (int c = 0; c < DK; ++c) {
                    y = fmaf(Kh[r * P + c], S0b[c * SP + j], y);
                    de = fmaf(-Bt[r * P + c], dSb[c * SP + j], de);
                }
                for (int s = 0; s < r; ++s) y = fmaf(Akk[r * CP + s], Ub[s * SP + j], y);
                for (int s = r; s < C; ++s) de = fmaf(-Aqb[s * CP + r], dOb[s * SP + j], de);
                Yb[r * SP + j] = y;
                dEb[r * SP + j] = de;
            }
            __syncthreads();
            // B3: E = T Y;  dY = T^T dE
            {
                const int r = rr, j = cl;
                float e = 0.f, dy = 0.f;
                for (int s = 0; s <= r; ++s) e = fmaf(Tm[r * CP + s], Yb[s * SP + j], e);
                for (int s = r; s < C; ++s) dy = fmaf(Tm[s * CP + r], dEb[s * SP + j], dy);
                Eb[r * SP + j] = e;
                dYb[r * SP + j] = dy;
            }
            __syncthreads();
            // B4: dU; dA; the [C][DK] sums; dG_C share; dS0 of this block
            {
                const int r = rr, j = cl;
                float du = 0.f;
#pragma unroll 4
                for (int c = 0; c < DK; ++c) du = fmaf(Kt[r * P + c], dSb[c * SP + j], du);
                for (int s = r; s < C; ++s) du = fmaf(Aqk[s * CP + r], dOb[s * SP + j], du);
                for (int s = r + 1; s < C; ++s) du = fmaf(Akk[s * CP + r], dYb[s * SP + j], du);
                if (r < n) {
                    const long long tok = tok_of(t0 + r), base = tok * DV;
                    dv[base + j0 + j] = from_f32<Tin>(wv * du);
                    if (w_kind == GDR_GATE_VECTOR) dw[base + j0 + j] = from_f32<Tin>(vv * du);
                    dw_row = fmaf(vv, du, dw_row);
                }
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = rr, s = cl + 16 * h2;
#pragma unroll
                for (int j = 0; j < DB; ++j) {
                    const float go = dOb[r * SP + j], gy = dYb[r * SP + j];
                    const float us = Ub[s * SP + j], es = Eb[s * SP + j];
                    aqk[h2] = fmaf(go, us, aqk[h2]);
                    aqb[h2] = fmaf(-go, es, aqb[h2]);
                    akk[h2] = fmaf(gy, us, akk[h2]);
                    akb[h2] = fmaf(-gy, es, akb[h2]);
                }
            }
#pragma unroll 4
            for (int j = 0; j < DB; ++j) {
                const int r = rr;
                const float go = dOb[r * SP + j], gy = dYb[r * SP + j];
                const float ur = Ub[r * SP + j], er = Eb[r * SP + j];
#pragma unroll
                for (int i = 0; i < NCI; ++i) {
                    const int c = cl + 16 * i;
                    const float s0 = S0b[c * SP + j], ds = dSb[c * SP + j];
                    xq[i] = fmaf(go, s0, xq[i]);
                    xk[i] = fmaf(gy, s0, xk[i]);
                    yk[i] = fmaf(ur, ds, yk[i]);
                    yb[i] = fmaf(-er, ds, yb[i]);
                }
            }
            if (tid < DK) {
#pragma unroll 4
                for (int j = 0; j < DB; ++j) gcp = fmaf(dSb[tid * SP + j], S0b[tid * SP + j], gcp);
            }
            for (int x = tid; x < DK * DB; x += NT) {
                const int c = x / DB, j = x % DB;
                float acc = egc[c] * dSb[c * SP + j];
                for (int r = 0; r < n; ++r) {
                    acc = fmaf(Qh[r * P + c], dOb[r * SP + j], acc);
                    acc = fmaf(Kh[r * P + c], dYb[r * SP + j], acc);
                }
                ds_run[soff + (size_t)c * DV + j0 + j] = acc;
            }
            __syncthreads();  // block's tiles consumed before the next block loads
        }

        // scalar write gate: one value per token
        if (w_kind == GDR_GATE_SCALAR) {
#pragma unroll
            for (int m = 8; m >= 1; m >>= 1) dw_row += __shfl_xor_sync(0xffffffffu, dw_row, m);
            if (cl == 0 && rr < n) dw[tok_of(t0 + rr)] = from_f32<Tin>(dw_row);
        }

        // gradient on G_C: e^G_C rowsum(dS_C S0) + colsum(Kt YK + Bt YB), taken
        // before the grams' shares join YK and YB (rows summed in a fixed order)
#pragma unroll
        for (int i = 0; i < NCI; ++i) {
            const int c = cl + 16 * i;
            gcr[rr * P + c] = Kt[rr * P + c] * yk[i] + Bt[rr * P + c] * yb[i];
        }
        // masked dA into the scratch (stage-B tiles are consumed)
        float* dAqk = scr;
        float* dAqb = scr + C * CP;
        float* dAkk = scr + 2 * C * CP;
        float* dAkb = scr + 3 * C * CP;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = rr, s = cl + 16 * h2;
            dAqk[r * CP + s] = s <= r ? aqk[h2] : 0.f;
            dAqb[r * CP + s] = s <= r ? aqb[h2] : 0.f;
            dAkk[r * CP + s] = s < r ? akk[h2] : 0.f;
            dAkb[r * CP + s] = s < r ? akb[h2] : 0.f;
        }
        __syncthreads();
        if (tid < DK) {
            float g = egc[tid] * gcp;
            for (int r = 0; r < C; ++r) g += gcr[r * P + tid];
            dgc[tid] = g;
        }

        // ---------------- stage C: the grams' gradients
        {
            const int r = rr;
            float pq[NCI], pk[NCI], qk_[NCI], qb_[NCI];
#pragma unroll
            for (int i = 0; i < NCI; ++i) pq[i] = pk[i] = qk_[i] = qb_[i] = 0.f;
            for (int s = 0; s < C; ++s) {
                const float gqk = dAqk[r * CP + s], gqb = dAqb[r * CP + s];
                const float gkk = dAkk[r * CP + s], gkb = dAkb[r * CP + s];
                const float tqk = dAqk[s * CP + r], tqb = dAqb[s * CP + r];
                const float tkk = dAkk[s * CP + r], tkb = dAkb[s * CP + r];
#pragma unroll
                for (int i = 0; i < NCI; ++i) {
                    const int c = cl + 16 * i;
                    const float kts = Kt[s * P + c], bts = Bt[s * P + c];
                    const float qhs = Qh[s * P + c], khs = Kh[s * P + c];
                    pq[i] = fmaf(gqk, kts, fmaf(gqb, bts, pq[i]));
                    pk[i] = fmaf(gkk, kts, fmaf(gkb, bts, pk[i]));
                    qk_[i] = fmaf(tqk, qhs, fmaf(tkk, khs, qk_[i]));
                    qb_[i] = fmaf(tqb, qhs, fmaf(tkb, khs, qb_[i]));
                }
            }
#pragma unroll
            for (int i = 0; i < NCI; ++i) {
                const float f = igc[cl + 16 * i];
                xq[i] = fmaf(f, pq[i], xq[i]);
                xk[i] = fmaf(f, pk[i], xk[i]);
                yk[i] = fmaf(f, qk_[i], yk[i]);
                yb[i] = fmaf(f, qb_[i], yb[i]);
            }
        }
        __syncthreads();  // dA reads done: the scratch becomes dG

        // ---------------- stage D: back to q, k, b and the decay
        float* dG = scr;
        {
            const int r = rr;
            float db_row = 0.f;
#pragma unroll
            for (int i = 0; i < NCI; ++i) {
                const int c = cl + 16 * i;
                float g = 0.f;
                if (r < n) {
                    const float gr = Gs[r * P + c], gc = Gs[(C - 1) * P + c];
                    const float eg = __expf(gr), et = __expf(gc - gr);
                    const float kt = Kt[r * P + c], bt = Bt[r * P + c];
                    const long long tok = tok_of(t0 + r), base = tok * DK;
                    dq[base + c] = from_f32<Tin>(eg * xq[i]);
                    dk[base + c] = from_f32<Tin>(fmaf(eg, xk[i], et * (yk[i] + Bs[r * P + c] * yb[i])));
                    const float dbv = kt * yb[i];
                    if (b_kind == GDR_GATE_VECTOR) db[base + c] = from_f32<Tin>(dbv);
                    db_row += dbv;
                    g = Qh[r * P + c] * xq[i] + Kh[r * P + c] * xk[i] - kt * yk[i] - bt * yb[i];
                    if (r == n - 1) g += dgc[c];
                }
                dG[r * P + c] = g;
            }
            if (b_kind == GDR_GATE_SCALAR) {
#pragma unroll
                for (int m = 8; m >= 1; m >>= 1) db_row += __shfl_xor_sync(0xffffffffu, db_row, m);
                if (cl == 0 && r < n) db[tok_of(t0 + r)] = from_f32<Tin>(db_row);
            }
        }
        __syncthreads();
        if (a_kind != GDR_GATE_ONE) {
            if (tid < DK) {  // d log a_r = sum_{r' >= r} dG_r';  da = d log a / a
                const int c = tid;
                float run = 0.f;
                for (int r = n - 1; r >= 0; --r) {
                    run += dG[r * P + c];
                    const long long tok = tok_of(t0 + r), base = tok * DK;
                    const float av = gate_value(a, a_kind, tok, base, c);
                    const float g = run / av;
                    if (a_kind == GDR_GATE_VECTOR) da[base + c] = from_f32<Tin>(g);
                    else dG[r * P + c] = g;
                }
            }
            if (a_kind == GDR_GATE_SCALAR) {
                __syncthreads();
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < NCI; ++i) s += dG[rr * P + cl + 16 * i];
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
static cudaError_t launch_backward_t(const gdr_desc& d, const void* const* in, const void* dout,
                                     const float* ds_final, float* hs, float* ds_run,
                                     void* const* grads, float* ds0, int* err_word,
                                     cudaStream_t st) {
    auto kern = backward_kernel<Tin, DK, DV>;
    const size_t smem = BwdSmem<DK>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((long long)d.B * d.H), BW_NT, smem, st>>>(
        d.T, d.H, (const Tin*)in[0], (const Tin*)in[1], (const Tin*)in[2], (const Tin*)in[3],
        (const Tin*)in[4], (const Tin*)in[5], (int)d.decay, (int)d.erase, (int)d.write,
        (const Tin*)dout, ds_final, hs, ds_run, (Tin*)grads[0], (Tin*)grads[1], (Tin*)grads[2],
        (Tin*)grads[3], (Tin*)grads[4], (Tin*)grads[5], ds0, err_word);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_backward_d(const gdr_desc& d, const void* const* in, const void* dout,
                                     const float* ds_final, float* hs, float* ds_run,
                                     void* const* grads, float* ds0, int* err_word,
                                     cudaStream_t st) {
#define GDR_BWD(DK_, DV_)                                                                    \
    if (d.dk == DK_ && d.dv == DV_)                                                          \
        return launch_backward_t<Tin, DK_, DV_>(d, in, dout, ds_final, hs, ds_run, grads, ds0, \
                                                err_word, st);
    GDR_BWD(128, 128)
    GDR_BWD(128, 64)
    GDR_BWD(64, 128)
    GDR_BWD(64, 64)
#undef GDR_BWD
    return cudaErrorInvalidValue;
}

size_t backward_workspace_bytes(const gdr_desc& d) {
    const size_t heads = (size_t)d.B * d.H;
    const size_t mat = (size_t)d.dk * d.dv * sizeof(float);
    const size_t n_chunks = ((size_t)d.T + BW_C - 1) / BW_C;
    return heads * mat * (n_chunks + 1);  // chunk-start states, then the running dS
}

cudaError_t launch_chunked_simt(const gdr_desc& d, const void* q, const void* k,
                                const void* v, const void* a, const void* b, const void* w,
                                const float* s0, void* o, float* s_final,
                                const int* cu_seqlens, int n_seqs, float* h_out,
                                int* err_word, cudaStream_t st);

// in = {q, k, v, a, b, w}; grads = {dq, dk, dv, da, db, dw}.
cudaError_t launch_backward(const gdr_desc& d, const void* const* in, const float* s0,
                            const void* dout, const float* ds_final, void* const* grads,
                            float* ds0, void* workspace, int* err_word, cudaStream_t st) {
    const size_t heads = (size_t)d.B * d.H;
    const size_t n_chunks = ((size_t)d.T + BW_C - 1) / BW_C;
    float* hs = static_cast<float*>(workspace);
    float* ds_run = hs + heads * n_chunks * d.dk * d.dv;
    if (d.T > 0) {
        gdr_desc f = d;
        f.chunk = BW_C;  // chunk-start states on the backward's chunk grid
        cudaError_t e = launch_chunked_simt(f, in[0], in[1], in[2], in[3], in[4], in[5], s0,
                                            nullptr, nullptr, nullptr, 0, hs, err_word, st);
        if (e != cudaSuccess) return e;
    }
    if (d.in_dtype == GDR_BF16)
        return launch_backward_d<__nv_bfloat16>(d, in, dout, ds_final, hs, ds_run, grads, ds0,
                                                err_word, st);
    return launch_backward_d<float>(d, in, dout, ds_final, hs, ds_run, grads, ds0, err_word, st);
}

}  // namespace gdr
