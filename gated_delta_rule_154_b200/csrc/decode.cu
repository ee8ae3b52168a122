// decode.cu -- single-token decode step of the gated delta rule.
//
// Per (batch, head), with the state S [dk, dv] float32 in HBM:
//     e_j   = sum_i a_i k_i S_ij                   (key read of the decayed state)
//     S_ij <- a_i S_ij - b_i k_i e_j + k_i w_j v_j  (decay, erase, write)
//     o_j   = sum_i q_i S_ij                        (read-out of the new state)
// FG^2-GDN page (gist.science 2604.19021), section 2 "Methodology", update
// rule, with Gated DeltaNet-2's decoupled erase/write gates (needhelp.icu,
// gates table).  The fixed-size state is the whole decode memory (Gated
// DeltaNet-2 page, "The attention bottleneck": O(1) decode memory).
//
// The step is bound by HBM: every state element is read once and written
// once, 8 bytes per element, against ~6 flops.  One CTA owns one head: its
// 256 threads load the whole 64 KB state into registers with 16-byte loads
// (each warp reads whole 512-byte rows), reduce e over the key axis (in
// registers, then across warps through shared memory), update in registers,
// store the new state with 16-byte stores, and reduce o the same way.
//
// Paged form (many sequences, one state pool): batch entry b reads and
// writes pool slot slot[b] instead of state b; an out-of-range slot is
// skipped and flagged in the device error word.
#include "common.cuh"

namespace gdr {

// Gate value without the FG2 form (the common instantiations keep exactly
// the plain staging code).
template <typename T>
__device__ __forceinline__ float plain_gate(const T* g, int kind, long long sidx,
                                            long long vbase, int c) {
    if (kind == GDR_GATE_ONE) return 1.0f;
    if (kind == GDR_GATE_SCALAR) return to_f32(g[sidx]);
    return to_f32(g[vbase + c]);
}

// PAGED: states come from a pool through slot[]; FG2: erase and/or write
// given as FG^2-GDN learning rates.  Both are compile-time so the plain
// step compiles to the plain code.
template <typename Tin, int DK, int DV, bool PAGED, bool FG2>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const Tin* __restrict__ a,
                   const Tin* __restrict__ b, const Tin* __restrict__ w,
                   int a_kind, int b_kind, int w_kind,
                   float* __restrict__ state, Tin* __restrict__ o, int H,
                   const int* __restrict__ slot, int n_slots, int* __restrict__ err_word) {
    constexpr int NT = 256;
    constexpr int TPR = DV / 4;     // threads per state row (one float4 each)
    constexpr int RS = NT / TPR;    // rows handled side by side
    constexpr int RPT = DK / RS;    // rows per thread
    static_assert(DV % 4 == 0 && NT % TPR == 0 && DK % RS == 0, "shape");

    __shared__ float qs[DK], ks[DK], as_[DK], bks[DK];
    __shared__ float us[DV];
    __shared__ __align__(16) float red[RS][DV];

    const int tid = threadIdx.x;
    const long long bh = blockIdx.x;  // (b * H + h)
    const int cg = tid % TPR;         // column group: columns 4cg .. 4cg+3
    const int rs = tid / TPR;         // row set: rows rs, rs + RS, ...

    long long sidx = bh;  // state of this (batch, head)
    if (PAGED) {
        const long long bi = bh / H;
        const int sl = slot[bi];
        if (sl < 0 || sl >= n_slots) {  // whole CTA agrees: skip, flag once
            if (tid == 0 && bh % H == 0) atomicOr(err_word, kErrIndex);
            return;
        }
        sidx = (long long)sl * H + bh % H;
    }
    float* S = state + sidx * (long long)DK * DV;

    // Issue the state loads first so they are in flight while the small
    // inputs are staged.
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
        s[r] = *reinterpret_cast<const float4*>(S + (size_t)(rs + RS * r) * DV + 4 * cg);

    for (int i = tid; i < DK; i += NT) {
        const long long vb = bh * DK;
        float kv = to_f32(k[vb + i]);
        float bv;
        if (FG2 && b_kind == GDR_GATE_FG2) {  // key sqrt(beta^k) k, erase gate 1
            kv *= sqrt_fast(fmaxf(to_f32(b[vb + i]), 0.f));
            bv = 1.f;
        } else {
            bv = plain_gate(b, b_kind, bh, vb, i);
        }
        qs[i] = to_f32(q[vb + i]);
        ks[i] = kv;
        as_[i] = plain_gate(a, a_kind, bh, vb, i);
        bks[i] = bv * kv;
    }
    for (int j = tid; j < DV; j += NT) {
        const long long vb = bh * DV;
        const float wv = (FG2 && w_kind == GDR_GATE_FG2) ? sqrt_fast(fmaxf(to_f32(w[vb + j]), 0.f))
                                                          : plain_gate(w, w_kind, bh, vb, j);
        us[j] = wv * to_f32(v[vb + j]);
    }
    __syncthreads();

    // e partial over this thread's rows.
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rs + RS * r;
        const float c = as_[i] * ks[i];
        e.x = fmaf(c, s[r].x, e.x);
        e.y = fmaf(c, s[r].y, e.y);
        e.z = fmaf(c, s[r].z, e.z);
        e.w = fmaf(c, s[r].w, e.w);
    }
    *reinterpret_cast<float4*>(&red[rs][4 * cg]) = e;
    __syncthreads();
    e = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int x = 0; x < RS; ++x) {
        const float4 p = *reinterpret_cast<const float4*>(&red[x][4 * cg]);
        e.x += p.x; e.y += p.y; e.z += p.z; e.w += p.w;
    }
    const float4 u = *reinterpret_cast<const float4*>(&us[4 * cg]);
    __syncthreads();  // everyone has read red[] before it is reused for o

    float4 op = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rs + RS * r;
        const float ai = as_[i], bki = bks[i], ki = ks[i], qi = qs[i];
        float4 n;
        n.x = fmaf(ai, s[r].x, fmaf(-bki, e.x, ki * u.x));
        n.y = fmaf(ai, s[r].y, fmaf(-bki, e.y, ki * u.y));
        n.z = fmaf(ai, s[r].z, fmaf(-bki, e.z, ki * u.z));
        n.w = fmaf(ai, s[r].w, fmaf(-bki, e.w, ki * u.w));
        *reinterpret_cast<float4*>(S + (size_t)i * DV + 4 * cg) = n;
        op.x = fmaf(qi, n.x, op.x);
        op.y = fmaf(qi, n.y, op.y);
        op.z = fmaf(qi, n.z, op.z);
        op.w = fmaf(qi, n.w, op.w);
    }
    *reinterpret_cast<float4*>(&red[rs][4 * cg]) = op;
    __syncthreads();
    if (rs == 0) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int x = 0; x < RS; ++x) {
            const float4 p = *reinterpret_cast<const float4*>(&red[x][4 * cg]);
            acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
        }
        Tin* od = o + bh * DV + 4 * cg;
        od[0] = from_f32<Tin>(acc.x);
        od[1] = from_f32<Tin>(acc.y);
        od[2] = from_f32<Tin>(acc.z);
        od[3] = from_f32<Tin>(acc.w);
    }
}

struct DecodeArgs {
    const void *q, *k, *v, *a, *b, *w;
    float* state;
    void* o;
    const int* slot;  // nullptr: state b for batch entry b
    int n_slots;
    int* err_word;
};

template <typename Tin, int DK, int DV, bool PAGED, bool FG2>
static cudaError_t launch_decode_k(const gdr_desc& d, const DecodeArgs& x, cudaStream_t stream) {
    const unsigned grid = (unsigned)((long long)d.B * d.H);
    decode_step_kernel<Tin, DK, DV, PAGED, FG2><<<grid, 256, 0, stream>>>(
        (const Tin*)x.q, (const Tin*)x.k, (const Tin*)x.v, (const Tin*)x.a, (const Tin*)x.b,
        (const Tin*)x.w, (int)d.decay, (int)d.erase, (int)d.write, x.state, (Tin*)x.o, d.H,
        x.slot, x.n_slots, x.err_word);
    return cudaGetLastError();
}

template <typename Tin, int DK, int DV>
static cudaError_t launch_decode_t(const gdr_desc& d, const DecodeArgs& x, cudaStream_t stream) {
    const bool fg2 = d.erase == GDR_GATE_FG2 || d.write == GDR_GATE_FG2;
    if (x.slot)
        return fg2 ? launch_decode_k<Tin, DK, DV, true, true>(d, x, stream)
                   : launch_decode_k<Tin, DK, DV, true, false>(d, x, stream);
    return fg2 ? launch_decode_k<Tin, DK, DV, false, true>(d, x, stream)
               : launch_decode_k<Tin, DK, DV, false, false>(d, x, stream);
}

template <typename Tin>
static cudaError_t launch_decode_d(const gdr_desc& d, const DecodeArgs& x, cudaStream_t stream) {
    if (d.dk == 128 && d.dv == 128) return launch_decode_t<Tin, 128, 128>(d, x, stream);
    if (d.dk == 128 && d.dv == 64) return launch_decode_t<Tin, 128, 64>(d, x, stream);
    if (d.dk == 64 && d.dv == 128) return launch_decode_t<Tin, 64, 128>(d, x, stream);
    return launch_decode_t<Tin, 64, 64>(d, x, stream);
}

cudaError_t launch_decode(const gdr_desc& d, const void* q, const void* k, const void* v,
                          const void* a, const void* b, const void* w, float* state,
                          void* o, const int* slot, int n_slots, int* err_word,
                          cudaStream_t stream) {
    const DecodeArgs x{q, k, v, a, b, w, state, o, slot, n_slots, err_word};
    if (d.in_dtype == GDR_BF16) return launch_decode_d<__nv_bfloat16>(d, x, stream);
    return launch_decode_d<float>(d, x, stream);
}

}  // namespace gdr
