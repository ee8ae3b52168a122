// segment.cu -- sequence-parallel prefill: a sequence is split into segments
// that run side by side, joined by an exclusive scan of their affine maps.
//
// The recurrence is affine in the state: over a segment, the state at its end
// is S_out = M S_in + N, where M = prod_t (I - (b_t*k_t) k_t^T) Diag(a_t)
// (dk x dk, the segment run from S_in = I with the writes switched off) and
// N the segment run from S_in = 0.  Chaining the segments' (M, N) in order
// gives every segment's start state, from which each segment is run again
// for its outputs.  Long-sequence scaling is what the FG^2-GDN page
// (gist.science 2604.19021) reports in section 4 "Experimental results"
// (efficiency); the segment maps are the product form of the rank-1
// Householder-like transitions of its section 2 update rule.
//
//   gdr_segment_maps        (M, N) of one segment per (batch, head)
//   gdr_segment_scan        start states and final state from the maps
//   gdr_forward_segmented   the whole prefill on one GPU: B x P segments as
//                           packed sequences, maps, scan, second pass
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace gdr {
namespace segment {

constexpr int D = 128;     // dk = dv
constexpr int NT = 256;

// cu[s] for s = b P + p: row b's segment p is tokens [p L, min((p+1) L, T)) of
// that row, L = ceil(T / P) rounded up to a multiple of 64 (the tensor-core
// kernel's chunk), in the [1, B T] view of the tokens.
__global__ void bounds_kernel(int* cu, int B, int T, int P, int L) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s > B * P) return;
    if (s == B * P) { cu[s] = B * T; return; }
    const int b = s / P, p = s % P;
    cu[s] = b * T + min(T, p * L);
}

// n_mats identity matrices of size d x d.
__global__ void identity_kernel(float* m, long long n_mats, int d) {
    const long long total = n_mats * d * d;
    for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
         x += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(x % ((long long)d * d));
        m[x] = (e / d == e % d) ? 1.0f : 0.0f;
    }
}

// One CTA per (batch, head): S = s0 (or 0); for each segment p in order,
// s_start[p] = S, then S = M_p S + N_p (float32, in shared memory); s_final =
// S.  Matrix (b, p, h) sits at (b * bstride + p * pstride + h) * d * d.
__global__ void __launch_bounds__(NT, 1)
scan_kernel(int P, int H, long long pstride, long long bstride, const float* __restrict__ m,
            const float* __restrict__ n, const float* __restrict__ s0, float* __restrict__ s_start,
            float* __restrict__ s_final) {
    extern __shared__ float4 smem4[];
    float* S = reinterpret_cast<float*>(smem4);   // [D][D]
    float* Ms = S + D * D;                        // [D][D]
    const int tid = threadIdx.x;
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const size_t mat = (size_t)D * D;
    for (int x = tid; x < D * D; x += NT) S[x] = s0 ? s0[(size_t)blockIdx.x * mat + x] : 0.f;
    // thread (i0, j0): rows 8 (tid / 16) .., columns 8 (tid % 16) ..
    const int i0 = 8 * (tid >> 4), j0 = 8 * (tid & 15);
    for (int p = 0; p < P; ++p) {
        const size_t off = ((size_t)b * bstride + (size_t)p * pstride + h) * mat;
        __syncthreads();   // S complete
        for (int x = tid; x < D * D; x += NT) {
            if (s_start) s_start[off + x] = S[x];
            Ms[x] = m[off + x];
        }
        __syncthreads();
        float acc[8][8];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[r][c] = n[off + (size_t)(i0 + r) * D + j0 + c];
        for (int k = 0; k < D; ++k) {
            float mv[8], sv[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) mv[r] = Ms[(i0 + r) * D + k];
            const float4 s_a = *reinterpret_cast<const float4*>(S + k * D + j0);
            const float4 s_b = *reinterpret_cast<const float4*>(S + k * D + j0 + 4);
            sv[0] = s_a.x; sv[1] = s_a.y; sv[2] = s_a.z; sv[3] = s_a.w;
            sv[4] = s_b.x; sv[5] = s_b.y; sv[6] = s_b.z; sv[7] = s_b.w;
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(mv[r], sv[c], acc[r][c]);
        }
        __syncthreads();   // every thread done reading S
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) S[(i0 + r) * D + j0 + c] = acc[r][c];
    }
    __syncthreads();
    if (s_final)
        for (int x = tid; x < D * D; x += NT) s_final[(size_t)blockIdx.x * mat + x] = S[x];
}

size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// blocks of 256 threads for a grid-stride loop over `total` elements
unsigned grid_for(long long total) {
    return (unsigned)std::max(1LL, std::min(1024LL, (total + 255) / 256));
}

size_t esize(const gdr_desc& d) { return d.in_dtype == GDR_BF16 ? 2 : 4; }

bool supported(const gdr_desc* d) { return d && d->dk == D && d->dv == D; }

}  // namespace segment
}  // namespace gdr

using namespace gdr::segment;

extern "C" {

size_t gdr_segment_maps_workspace_size(const gdr_desc* d) {
    if (!supported(d) || d->B < 1 || d->T < 0 || d->H < 1) return 0;
    const size_t th = (size_t)d->B * d->T * d->H;
    return align16(th * esize(*d)) + align16(th * d->dv * esize(*d));
}

gdr_status gdr_segment_maps(const gdr_desc* d, const void* q, const void* k, const void* v,
                            const void* a, const void* b, const void* w, float* m_out,
                            float* n_out, void* workspace, size_t ws_bytes,
                            gdr_stream_t stream) {
    if (!d || !m_out || !n_out) return GDR_ERR_INVALID_ARG;
    if (!supported(d)) return GDR_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(m_out) | reinterpret_cast<uintptr_t>(n_out)) & 15u)
        return GDR_ERR_INVALID_ARG;
    const size_t need = gdr_segment_maps_workspace_size(d);
    if (!workspace || ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return GDR_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t th = (size_t)d->B * d->T * d->H;
    uint8_t* zeros = static_cast<uint8_t*>(workspace);          // write gate 0, [B, T, H]
    uint8_t* o_scr = zeros + align16(th * esize(*d));           // discarded outputs
    const long long n_mats = (long long)d->B * d->H;
    identity_kernel<<<grid_for(n_mats * D * D), 256, 0, st>>>(m_out, n_mats, D);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    if (th > 0 && cudaMemsetAsync(zeros, 0, th * esize(*d), st) != cudaSuccess)
        return GDR_ERR_CUDA;
    // M: from S = I with every write switched off (a scalar write gate of 0)
    gdr_desc dm = *d;
    dm.write = GDR_GATE_SCALAR;
    gdr_status s = gdr_forward_chunked(&dm, q, k, v, a, b, zeros, m_out, o_scr, m_out, nullptr,
                                       0, stream);
    if (s != GDR_OK) return s;
    // N: from S = 0
    return gdr_forward_chunked(d, q, k, v, a, b, w, nullptr, o_scr, n_out, nullptr, 0, stream);
}

gdr_status gdr_segment_scan(int n_segments, int B, int H, int dk, int dv, long long seg_stride,
                            long long batch_stride, const float* m, const float* n,
                            const float* s0, float* s_start, float* s_final,
                            gdr_stream_t stream) {
    if (n_segments < 1 || B < 1 || H < 1 || !m || !n) return GDR_ERR_INVALID_ARG;
    if (dk != D || dv != D) return GDR_ERR_UNSUPPORTED;
    if (seg_stride < 0 || batch_stride < 0) return GDR_ERR_INVALID_ARG;
    const uintptr_t any = reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(n) |
                          reinterpret_cast<uintptr_t>(s0) | reinterpret_cast<uintptr_t>(s_start) |
                          reinterpret_cast<uintptr_t>(s_final);
    if (any & 15u) return GDR_ERR_INVALID_ARG;
    const size_t smem = 2 * (size_t)D * D * sizeof(float);
    if (cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GDR_ERR_CUDA;
    scan_kernel<<<(unsigned)(B * H), NT, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        n_segments, H, seg_stride, batch_stride, m, n, s0, s_start, s_final);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

size_t gdr_segmented_workspace_size(const gdr_desc* d, int n_segments) {
    if (!supported(d) || n_segments < 1 || d->B < 1 || d->T < 0 || d->H < 1) return 0;
    const size_t mats = (size_t)d->B * n_segments * d->H * D * D * sizeof(float);
    const size_t th = (size_t)d->B * d->T * d->H;
    return align16(((size_t)d->B * n_segments + 1) * sizeof(int)) + align16(th * esize(*d)) +
           3 * mats;
}

gdr_status gdr_forward_segmented(const gdr_desc* d, int n_segments, const void* q,
                                 const void* k, const void* v, const void* a, const void* b,
                                 const void* w, const float* s0, void* o, float* s_final,
                                 void* workspace, size_t ws_bytes, gdr_stream_t stream) {
    if (!d || n_segments < 1) return GDR_ERR_INVALID_ARG;
    if (!supported(d)) return GDR_ERR_UNSUPPORTED;
    if (n_segments == 1 || d->T == 0)
        return gdr_forward_chunked(d, q, k, v, a, b, w, s0, o, s_final, nullptr, 0, stream);
    if ((long long)d->B * n_segments * d->H > 0x7fffffffLL) return GDR_ERR_INVALID_ARG;
    const size_t need = gdr_segmented_workspace_size(d, n_segments);
    if (!workspace || ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return GDR_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int P = n_segments, nseq = d->B * P;
    const size_t th = (size_t)d->B * d->T * d->H;
    const size_t mats = (size_t)nseq * d->H * D * D * sizeof(float);
    uint8_t* p8 = static_cast<uint8_t*>(workspace);
    int* cu = reinterpret_cast<int*>(p8);
    p8 += align16(((size_t)nseq + 1) * sizeof(int));
    uint8_t* zeros = p8;
    p8 += align16(th * esize(*d));
    float* M = reinterpret_cast<float*>(p8);
    float* N = reinterpret_cast<float*>(p8 + mats);
    float* S = reinterpret_cast<float*>(p8 + 2 * mats);
    const int L = (((d->T + P - 1) / P) + 63) / 64 * 64;
    bounds_kernel<<<(nseq + 1 + 255) / 256, 256, 0, st>>>(cu, d->B, d->T, P, L);
    identity_kernel<<<grid_for((long long)nseq * d->H * D * D), 256, 0, st>>>(
        M, (long long)nseq * d->H, D);
    if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    if (cudaMemsetAsync(zeros, 0, th * esize(*d), st) != cudaSuccess) return GDR_ERR_CUDA;
    // the B rows' segments as packed sequences of one [1, B T] row; o holds
    // the first two passes' (discarded) outputs
    gdr_desc dp = *d;
    dp.B = 1;
    dp.T = d->B * d->T;
    gdr_desc dm = dp;
    dm.write = GDR_GATE_SCALAR;
    gdr_status s = gdr_forward_varlen(&dm, cu, nseq, q, k, v, a, b, zeros, M, o, M, nullptr, 0,
                                      stream);
    if (s != GDR_OK) return s;
    s = gdr_forward_varlen(&dp, cu, nseq, q, k, v, a, b, w, nullptr, o, N, nullptr, 0, stream);
    if (s != GDR_OK) return s;
    s = gdr_segment_scan(P, d->B, d->H, D, D, d->H, (long long)P * d->H, M, N, s0, S, s_final,
                         stream);
    if (s != GDR_OK) return s;
    return gdr_forward_varlen(&dp, cu, nseq, q, k, v, a, b, w, S, o, nullptr, nullptr, 0, stream);
}

}  // extern "C"
