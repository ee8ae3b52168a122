// chunked_simt.cu -- chunkwise-parallel gated delta rule, float32 CUDA-core
// kernel.  This is the kernel for float32 inputs (where the products must stay
// in float32 to hold a 1e-4 error budget) and for shapes the tensor-core
// kernel does not take.
//
// Chunked form (per chunk of n <= C tokens, state S0 at the chunk start,
// G_r = sum_{i<=r} log a_i per key channel, U = w*V):
//   A_kk[r,s] = sum_c k_rc k_sc exp(G_rc - G_sc)          (s <  r)
//   A_kb[r,s] = sum_c k_rc b_sc k_sc exp(G_rc - G_sc)     (s <  r)
//   A_qk[r,s] = sum_c q_rc k_sc exp(G_rc - G_sc)          (s <= r)
//   A_qb[r,s] = sum_c q_rc b_sc k_sc exp(G_rc - G_sc)     (s <= r)
//   E  = (I + A_kb)^{-1} (Kh S0 + A_kk U),   Kh = exp(G) * K
//   O  = Qh S0 + A_qk U - A_qb E,            Qh = exp(G) * Q
//   S_C = exp(G_C) * S0 + Kt^T U - Bt^T E,   Kt = exp(G_C - G) * K, Bt = b * Kt
// Row r of E is the key read e_r = S'_r^T k_r of token r.  This is the WY /
// UT-transform evaluation the FG^2-GDN page (gist.science 2604.19021) names in
// section 2 "Methodology" (rank-1 Householder structure kept for WY chunked
// training) and section 3 (DPLR structure, KDA-style chunked kernels); the
// algebra is derived from the update rule of section 2.
//
// Every exponent here is a sum of log-decays over a run of tokens taken with
// its sign, so it is <= 0: no factor can overflow, whatever the decay.  The
// gram sums take one exp per term (the kernel trades speed for that range);
// the tensor-core kernel factorises instead.
//
// One CTA owns one (batch, head, block of DVB value columns) and walks the
// chunks in order, keeping its [dk, DVB] slice of S in shared memory.  The
// columns of S evolve independently (the transition multiplies from the
// left), so value-column blocks need no communication.
#include "common.cuh"

namespace gdr {

template <int DK, int DVB, int C>
struct SimtSmem {
    static constexpr int P = DK + 1;   // padded row stride of [C][DK] tiles
    static constexpr int CP = C + 1;   // padded row stride of [C][C] tiles
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + C * P;
    static constexpr int kG = kK + C * P;
    static constexpr int kB = kG + C * P;
    static constexpr int kS = kB + C * P;
    static constexpr int kU = kS + DK * DVB;
    static constexpr int kE = kU + C * DVB;
    static constexpr int kAkk = kE + C * DVB;
    static constexpr int kAkb = kAkk + C * CP;
    static constexpr int kAqk = kAkb + C * CP;
    static constexpr int kAqb = kAqk + C * CP;
    static constexpr int kGl = kAqb + C * CP;
    static constexpr int floats = kGl + DK;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename Tin, int DK, int DV, int C, int DVB>
__global__ void __launch_bounds__(256)
chunked_simt_kernel(int B, int T, int H,
                    const Tin* __restrict__ q, const Tin* __restrict__ k,
                    const Tin* __restrict__ v, const Tin* __restrict__ a,
                    const Tin* __restrict__ b, const Tin* __restrict__ w,
                    int a_kind, int b_kind, int w_kind,
                    const float* __restrict__ s0, Tin* __restrict__ o,
                    float* __restrict__ s_final, const int* __restrict__ cu_seqlens,
                    int* __restrict__ err_word) {
    constexpr int NT = 256;
    constexpr int SL = NT / DVB;  // s-slices per column in the triangular solve
    static_assert(SL == 8 || SL == 16, "DVB must be 32 or 16");
    using L = SimtSmem<DK, DVB, C>;
    constexpr int P = L::P, CP = L::CP;

    extern __shared__ float sm[];
    float* Qs = sm + L::kQ;   // q, then Qh
    float* Ks = sm + L::kK;   // k, then Kh
    float* Gs = sm + L::kG;   // cumulative log decay, then Kt
    float* Bs = sm + L::kB;   // erase gate, then Bt
    float* Ss = sm + L::kS;   // state slice [DK][DVB]
    float* Us = sm + L::kU;   // w*v [C][DVB]
    float* Es = sm + L::kE;   // key reads [C][DVB]
    float* Akk = sm + L::kAkk;
    float* Akb = sm + L::kAkb;
    float* Aqk = sm + L::kAqk;
    float* Aqb = sm + L::kAqb;
    float* Gl = sm + L::kGl;  // G at the chunk's last token, per channel

    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int hi = bh % H;
    // this CTA's tokens: [tb, tb + len) of batch row bi (packed sequences: one
    // batch row; a range outside the tensor is reported and skipped)
    int bi, tb, len;
    if (!seq_range(cu_seqlens, bh / H, T, bi, tb, len)) {
        if (tid == 0 && blockIdx.y == 0) atomicOr(err_word, kErrIndex);
        return;
    }
    const int j0 = blockIdx.y * DVB;

    const size_t soff = (size_t)bh * DK * DV;
    for (int x = tid; x < DK * DVB; x += NT) {
        const int c = x / DVB, j = x % DVB;
        Ss[x] = s0 ? s0[soff + (size_t)c * DV + j0 + j] : 0.0f;
    }

    for (int t0 = 0; t0 < len; t0 += C) {
        const int n = min(C, len - t0);
        __syncthreads();  // previous chunk finished with every buffer

        // ---- load the chunk; padded tokens act as a = 1, k = q = v = 0
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f;
            if (r < n) {
                const long long tok = ((long long)bi * T + tb + t0 + r) * H + hi;
                const long long base = tok * DK;
                qv = to_f32(q[base + c]);
                kv = to_f32(k[base + c]);
                bv = gate_value(b, b_kind, tok, base, c);
                if (b_kind == GDR_GATE_FG2) {  // key sqrt(beta^k) k, erase gate 1
                    kv *= bv;
                    bv = 1.f;
                }
                gv = a_kind == GDR_GATE_ONE ? 0.f
                                            : safe_log_decay(gate_value(a, a_kind, tok, base, c));
            }
            Qs[r * P + c] = qv;
            Ks[r * P + c] = kv;
            Bs[r * P + c] = bv;
            Gs[r * P + c] = gv;
        }
        for (int x = tid; x < C * DVB; x += NT) {
            const int r = x / DVB, j = x % DVB;
            float u = 0.f;
            if (r < n) {
                const long long tok = ((long long)bi * T + tb + t0 + r) * H + hi;
                const long long base = tok * DV;
                u = gate_value(w, w_kind, tok, base, j0 + j) * to_f32(v[base + j0 + j]);
            }
            Us[x] = u;
        }
        __syncthreads();

        // ---- cumulative log decay within the chunk
        for (int c = tid; c < DK; c += NT) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                run += Gs[r * P + c];
                Gs[r * P + c] = run;
            }
            Gl[c] = run;
        }
        __syncthreads();

        // ---- gram matrices over the lower triangle (s <= r)
        constexpr int NPAIR = C * (C + 1) / 2;
        for (int p = tid; p < NPAIR; p += NT) {
            int r = (int)((sqrtf(8.0f * p + 1.0f) - 1.0f) * 0.5f);
            while (r * (r + 1) / 2 > p) --r;
            while ((r + 1) * (r + 2) / 2 <= p) ++r;
            const int s = p - r * (r + 1) / 2;
            float kk = 0.f, kb = 0.f, qk = 0.f, qb = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) {
                const float f = __expf(Gs[r * P + c] - Gs[s * P + c]);
                const float ks = Ks[s * P + c] * f;
                const float bks = Bs[s * P + c] * ks;
                const float kr = Ks[r * P + c], qr = Qs[r * P + c];
                kk = fmaf(kr, ks, kk);
                kb = fmaf(kr, bks, kb);
                qk = fmaf(qr, ks, qk);
                qb = fmaf(qr, bks, qb);
            }
            Akk[r * CP + s] = (s < r) ? kk : 0.f;
            Akb[r * CP + s] = (s < r) ? kb : 0.f;
            Aqk[r * CP + s] = qk;
            Aqb[r * CP + s] = qb;
        }
        __syncthreads();

        // ---- scaled operands, in place: Qh, Kh, Kt, Bt
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            const float g = Gs[r * P + c];
            const float eg = __expf(g);
            const float et = __expf(Gl[c] - g);
            const float kv = Ks[r * P + c];
            Qs[r * P + c] *= eg;
            Ks[r * P + c] = kv * eg;
            Gs[r * P + c] = kv * et;
            Bs[r * P + c] = Bs[r * P + c] * kv * et;
        }
        __syncthreads();

        // ---- right-hand side: Kh S0 + A_kk U  (into Es)
        for (int x = tid; x < C * DVB; x += NT) {
            const int r = x / DVB, j = x % DVB;
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(Ks[r * P + c], Ss[c * DVB + j], acc);
            for (int s = 0; s < r; ++s) acc = fmaf(Akk[r * CP + s], Us[s * DVB + j], acc);
            Es[x] = acc;
        }
        __syncthreads();

        // ---- forward substitution: E[r] -= sum_{s<r} A_kb[r,s] E[s]
        {
            const int j = tid / SL, sl = tid % SL;  // one warp owns 32/SL columns
            for (int r = 1; r < n; ++r) {
                float part = 0.f;
                for (int s = sl; s < r; s += SL) part = fmaf(Akb[r * CP + s], Es[s * DVB + j], part);
#pragma unroll
                for (int m = 1; m < SL; m <<= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
                if (sl == 0) Es[r * DVB + j] -= part;
                __syncwarp();
            }
        }
        __syncthreads();

        // ---- outputs: O = Qh S0 + A_qk U - A_qb E
        for (int x = tid; x < C * DVB; x += NT) {
            const int r = x / DVB, j = x % DVB;
            if (r >= n) continue;
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(Qs[r * P + c], Ss[c * DVB + j], acc);
            for (int s = 0; s <= r; ++s)
                acc = fmaf(Aqk[r * CP + s], Us[s * DVB + j],
                           fmaf(-Aqb[r * CP + s], Es[s * DVB + j], acc));
            const long long tok = ((long long)bi * T + tb + t0 + r) * H + hi;
            o[tok * DV + j0 + j] = from_f32<Tin>(acc);
        }
        __syncthreads();

        // ---- state: S = exp(G_C) S0 + Kt^T U - Bt^T E
        for (int x = tid; x < DK * DVB; x += NT) {
            const int c = x / DVB, j = x % DVB;
            float acc = __expf(Gl[c]) * Ss[x];
            for (int s = 0; s < n; ++s)
                acc = fmaf(Gs[s * P + c], Us[s * DVB + j],
                           fmaf(-Bs[s * P + c], Es[s * DVB + j], acc));
            Ss[x] = acc;
        }
    }
    __syncthreads();
    if (s_final) {
        for (int x = tid; x < DK * DVB; x += NT) {
            const int c = x / DVB, j = x % DVB;
            s_final[soff + (size_t)c * DV + j0 + j] = Ss[x];
        }
    }
}

struct SimtArgs {
    const void *q, *k, *v, *a, *b, *w;
    const float* s0;
    void* o;
    float* s_final;
    const int* cu_seqlens;  // nullptr: batch rows as sequences
    int n_seqs;
    int* err_word;
};

template <typename Tin, int DK, int DV, int C, int DVB>
static cudaError_t launch_simt_t(const gdr_desc& d, const SimtArgs& x, cudaStream_t st) {
    auto kern = chunked_simt_kernel<Tin, DK, DV, C, DVB>;
    const size_t smem = SimtSmem<DK, DVB, C>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const long long nseq = x.cu_seqlens ? x.n_seqs : d.B;
    dim3 grid((unsigned)(nseq * d.H), DV / DVB);
    kern<<<grid, 256, smem, st>>>(d.B, d.T, d.H, (const Tin*)x.q, (const Tin*)x.k,
                                  (const Tin*)x.v, (const Tin*)x.a, (const Tin*)x.b,
                                  (const Tin*)x.w, (int)d.decay, (int)d.erase, (int)d.write,
                                  x.s0, (Tin*)x.o, x.s_final, x.cu_seqlens, x.err_word);
    return cudaGetLastError();
}

template <typename Tin, int DK, int DV>
static cudaError_t launch_simt_c(const gdr_desc& d, const SimtArgs& x, cudaStream_t st) {
    switch (d.chunk) {
        case 16: return launch_simt_t<Tin, DK, DV, 16, 32>(d, x, st);
        case 32: return launch_simt_t<Tin, DK, DV, 32, 32>(d, x, st);
        default:
            if (DK == 128) return launch_simt_t<Tin, DK, DV, 64, 16>(d, x, st);
            return launch_simt_t<Tin, DK, DV, 64, 32>(d, x, st);
    }
}

template <typename Tin>
static cudaError_t launch_simt_d(const gdr_desc& d, const SimtArgs& x, cudaStream_t st) {
    if (d.dk == 128 && d.dv == 128) return launch_simt_c<Tin, 128, 128>(d, x, st);
    if (d.dk == 128 && d.dv == 64) return launch_simt_c<Tin, 128, 64>(d, x, st);
    if (d.dk == 64 && d.dv == 128) return launch_simt_c<Tin, 64, 128>(d, x, st);
    return launch_simt_c<Tin, 64, 64>(d, x, st);
}

cudaError_t launch_chunked_simt(const gdr_desc& d, const void* q, const void* k,
                                const void* v, const void* a, const void* b, const void* w,
                                const float* s0, void* o, float* s_final,
                                const int* cu_seqlens, int n_seqs, int* err_word,
                                cudaStream_t st) {
    const SimtArgs x{q, k, v, a, b, w, s0, o, s_final, cu_seqlens, n_seqs, err_word};
    if (d.in_dtype == GDR_BF16) return launch_simt_d<__nv_bfloat16>(d, x, st);
    return launch_simt_d<float>(d, x, st);
}

}  // namespace gdr
