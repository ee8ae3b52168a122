// common.cuh -- small device helpers shared by the gated delta-rule kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdr.h"

namespace gdr {

// Device error word bits.  A kernel that detects a problem ORs its bit into
// the word it was given; gdr_last_device_error() turns the bits into a status.
enum : int { kErrTimeout = 1, kErrRange = 2, kErrIndex = 4 };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Square root to about 1 ulp in one SFU op (non-negative input; ftz).  The
// IEEE-rounded sqrtf brings a slow-path routine into the kernel that
// measurably slowed the decode step even where it never runs.
__device__ __forceinline__ float sqrt_fast(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Value of gate `g` of kind `kind` for channel c of the token/head whose
// scalar index is `sidx` and whose vector row starts at `vbase`.
template <typename T>
__device__ __forceinline__ float gate_value(const T* g, int kind, long long sidx,
                                            long long vbase, int c) {
    if (kind == GDR_GATE_ONE) return 1.0f;
    if (kind == GDR_GATE_SCALAR) return to_f32(g[sidx]);
    if (kind == GDR_GATE_FG2) return sqrt_fast(fmaxf(to_f32(g[vbase + c]), 0.0f));  // sqrt(beta)
    return to_f32(g[vbase + c]);
}

// Token range of one CTA's sequence: tokens [tb, tb + len) of batch row bi.
// Without cu_seqlens, sequence `seq` is batch row `seq` (all T tokens);
// with it (packed sequences in one batch row), sequence `seq` spans
// [cu[seq], cu[seq + 1]).  Returns false for a range outside [0, T], which
// the caller reports and skips.
__device__ __forceinline__ bool seq_range(const int* cu, int seq, int T, int& bi, int& tb,
                                          int& len) {
    if (!cu) {
        bi = seq;
        tb = 0;
        len = T;
        return true;
    }
    bi = 0;
    tb = cu[seq];
    const int te = cu[seq + 1];
    len = te - tb;
    return tb >= 0 && te >= tb && te <= T;
}

// Natural log of a decay value with a floor at log(FLT_MIN) so that a = 0
// (or a denormal) behaves as a full reset instead of producing -inf.
__device__ __forceinline__ float safe_log_decay(float a) {
    return fmaxf(logf(a), -87.0f);
}

}  // namespace gdr
