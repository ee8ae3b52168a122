// gdr_api.cu -- the C ABI of libgdr.so: argument checks, kernel choice,
// device error word.  Declarations and contracts are in include/gdr.h.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace gdr {
cudaError_t launch_decode(const gdr_desc& d, const void* q, const void* k, const void* v,
                          const void* a, const void* b, const void* w, float* state,
                          void* o, const int* slot, int n_slots, int* err_word,
                          cudaStream_t stream);
cudaError_t launch_chunked_simt(const gdr_desc& d, const void* q, const void* k,
                                const void* v, const void* a, const void* b, const void* w,
                                const float* s0, void* o, float* s_final,
                                const int* cu_seqlens, int n_seqs, int* err_word,
                                cudaStream_t st);
bool chunked_tc_supports(const gdr_desc& d);
size_t backward_workspace_bytes(const gdr_desc& d, int n_seqs);
cudaError_t launch_backward(const gdr_desc& d, const int* cu_seqlens, int n_seqs,
                            const void* const* in, const float* s0, const void* dout,
                            const float* ds_final, void* const* grads, float* ds0,
                            void* workspace, int* err_word, cudaStream_t st);
cudaError_t launch_chunked_tc(const gdr_desc& d, const void* q, const void* k, const void* v,
                              const void* a, const void* b, const void* w, const float* s0,
                              void* o, float* s_final, int* err_word, bool skip_signal,
                              const int* cu_seqlens, int n_seqs, cudaStream_t st);
}  // namespace gdr

// One error word per device (each device holds its own copy of the symbol).
static __device__ int g_gdr_error_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::atomic<int> g_test_skip_signal{0};  // gdr_test_skip_signal, consumed by one launch
int* g_err_ptr[kMaxDevices];

// Device address of this device's error word (looked up once per device).
cudaError_t error_word(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gdr_error_word);
        if (e != cudaSuccess) return e;
        g_err_ptr[dev] = static_cast<int*>(p);
    }
    *out = g_err_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_gate(int g) { return g == GDR_GATE_ONE || g == GDR_GATE_SCALAR || g == GDR_GATE_VECTOR; }
bool valid_gate_beta(int g) { return valid_gate(g) || g == GDR_GATE_FG2; }  // erase, write

// Checks shared by both entry points; `T_axis` tells whether T is part of the
// tensor shapes (prefill) or fixed to 1 (decode).
gdr_status check_desc(const gdr_desc* d) {
    if (!d) return GDR_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->T < 0) return GDR_ERR_INVALID_ARG;
    if ((long long)d->B * d->H > 0x7fffffffLL) return GDR_ERR_INVALID_ARG;
    if ((long long)d->B * d->T > (1LL << 40)) return GDR_ERR_INVALID_ARG;
    if (!(d->dk == 64 || d->dk == 128) || !(d->dv == 64 || d->dv == 128))
        return GDR_ERR_INVALID_ARG;
    if (!(d->chunk == 16 || d->chunk == 32 || d->chunk == 64)) return GDR_ERR_INVALID_ARG;
    if (!(d->in_dtype == GDR_F32 || d->in_dtype == GDR_BF16)) return GDR_ERR_INVALID_ARG;
    if (!valid_gate(d->decay) || !valid_gate_beta(d->erase) || !valid_gate_beta(d->write))
        return GDR_ERR_INVALID_ARG;
    return GDR_OK;
}

gdr_status check_ptr(const void* p, bool required) {
    if (!p) return required ? GDR_ERR_INVALID_ARG : GDR_OK;
    return aligned16(p) ? GDR_OK : GDR_ERR_INVALID_ARG;
}

gdr_status check_inputs(const gdr_desc* d, bool have_tokens, const void* q, const void* k,
                        const void* v, const void* a, const void* b, const void* w,
                        const void* o) {
    gdr_status s;
    if ((s = check_ptr(q, have_tokens)) != GDR_OK) return s;
    if ((s = check_ptr(k, have_tokens)) != GDR_OK) return s;
    if ((s = check_ptr(v, have_tokens)) != GDR_OK) return s;
    if ((s = check_ptr(o, have_tokens)) != GDR_OK) return s;
    if ((s = check_ptr(a, have_tokens && d->decay != GDR_GATE_ONE)) != GDR_OK) return s;
    if ((s = check_ptr(b, have_tokens && d->erase != GDR_GATE_ONE)) != GDR_OK) return s;
    if ((s = check_ptr(w, have_tokens && d->write != GDR_GATE_ONE)) != GDR_OK) return s;
    return GDR_OK;
}

// The float32 kernel takes every (dk, dv, chunk) the checks admit.
bool simt_supports(const gdr_desc&) { return true; }

}  // namespace

extern "C" {

int gdr_version(void) { return 0x000100; }

const char* gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
        case GDR_ERR_RANGE: return "GDR_ERR_RANGE";
    }
    return "GDR_UNKNOWN_STATUS";
}

}  // extern "C"

namespace {
// The automatic sequence split of gdr_forward_chunked: when B * H heads leave
// at least three quarters of the B200's 148 SMs idle, each sequence is cut
// into P = 148 / (B * H) segments that run side by side (their affine maps,
// a scan, a second pass: three passes of T / P tokens instead of one of T),
// provided every segment keeps at least 64 chunks of 64 tokens.
constexpr int kSMs = 148;
int auto_segments(const gdr_desc& d) {
    if (!(d.in_dtype == GDR_BF16 && d.dk == 128 && d.dv == 128 && d.chunk == 64)) return 1;
    const long long P = kSMs / ((long long)d.B * d.H);
    if (P < 4 || (long long)d.T < 4096LL * P) return 1;
    return (int)P;
}
}  // namespace

extern "C" {

size_t gdr_workspace_size(const gdr_desc* d) {
    if (check_desc(d) != GDR_OK) return 0;
    const int P = auto_segments(*d);
    // every kernel keeps its intermediates on chip; only the split needs room
    return P > 1 ? gdr_segmented_workspace_size(d, P) : 0;
}

namespace {
gdr_status forward_impl(const gdr_desc* d, const int* cu_seqlens, int n_seqs, const void* q,
                        const void* k, const void* v, const void* a, const void* b,
                        const void* w, const float* s0, void* o, float* s_final,
                        void* workspace, size_t ws_bytes, gdr_stream_t stream) {
    gdr_status s = check_desc(d);
    if (s != GDR_OK) return s;
    const bool have_tokens = d->T > 0;
    if ((s = check_inputs(d, have_tokens, q, k, v, a, b, w, o)) != GDR_OK) return s;
    if ((s = check_ptr(s0, false)) != GDR_OK) return s;
    if ((s = check_ptr(s_final, false)) != GDR_OK) return s;
    // packed sequences never split; a NULL workspace keeps the one-pass kernel
    const size_t need = cu_seqlens ? 0 : gdr_workspace_size(d);
    if (need > 0 && workspace != nullptr && ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return GDR_ERR_INVALID_ARG;

    if (d->T == 0 && s_final == nullptr) return GDR_OK;  // nothing to compute or write
    if (need > 0 && workspace != nullptr)
        return gdr_forward_segmented(d, auto_segments(*d), q, k, v, a, b, w, s0, o, s_final,
                                     workspace, ws_bytes, stream);

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int* err = nullptr;
    if (error_word(&err) != cudaSuccess) return GDR_ERR_CUDA;
    cudaError_t e;
    if (gdr::chunked_tc_supports(*d)) {
        const bool skip = g_test_skip_signal.exchange(0) != 0;
        e = gdr::launch_chunked_tc(*d, q, k, v, a, b, w, s0, o, s_final, err, skip, cu_seqlens,
                                   n_seqs, st);
    } else if (simt_supports(*d)) {
        e = gdr::launch_chunked_simt(*d, q, k, v, a, b, w, s0, o, s_final, cu_seqlens, n_seqs,
                                     err, st);
    } else {
        return GDR_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}
}  // namespace

gdr_status gdr_forward_chunked(const gdr_desc* d, const void* q, const void* k, const void* v,
                               const void* a, const void* b, const void* w, const float* s0,
                               void* o, float* s_final, void* workspace, size_t ws_bytes,
                               gdr_stream_t stream) {
    return forward_impl(d, nullptr, 0, q, k, v, a, b, w, s0, o, s_final, workspace, ws_bytes,
                        stream);
}

gdr_status gdr_forward_varlen(const gdr_desc* d, const int* cu_seqlens, int n_seqs,
                              const void* q, const void* k, const void* v, const void* a,
                              const void* b, const void* w, const float* s0, void* o,
                              float* s_final, void* workspace, size_t ws_bytes,
                              gdr_stream_t stream) {
    if (!d || d->B != 1 || n_seqs < 1) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr || reinterpret_cast<uintptr_t>(cu_seqlens) % 4 != 0)
        return GDR_ERR_INVALID_ARG;
    if ((long long)n_seqs * d->H > 0x7fffffffLL) return GDR_ERR_INVALID_ARG;
    if (d->T == 0 && s_final == nullptr) {
        gdr_status s = check_desc(d);
        return s;
    }
    return forward_impl(d, cu_seqlens, n_seqs, q, k, v, a, b, w, s0, o, s_final, workspace,
                        ws_bytes, stream);
}

gdr_status gdr_decode_step(const gdr_desc* d, const void* q, const void* k, const void* v,
                           const void* a, const void* b, const void* w, float* state, void* o,
                           gdr_stream_t stream) {
    gdr_status s = check_desc(d);
    if (s != GDR_OK) return s;
    if (d->T != 1) return GDR_ERR_INVALID_ARG;
    if ((s = check_inputs(d, true, q, k, v, a, b, w, o)) != GDR_OK) return s;
    if ((s = check_ptr(state, true)) != GDR_OK) return s;
    cudaError_t e = gdr::launch_decode(*d, q, k, v, a, b, w, state, o, nullptr, 0, nullptr,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status gdr_decode_step_paged(const gdr_desc* d, const void* q, const void* k, const void* v,
                                 const void* a, const void* b, const void* w, float* state_pool,
                                 const int* slot, int n_slots, void* o, gdr_stream_t stream) {
    gdr_status s = check_desc(d);
    if (s != GDR_OK) return s;
    if (d->T != 1 || n_slots < 1) return GDR_ERR_INVALID_ARG;
    if ((s = check_inputs(d, true, q, k, v, a, b, w, o)) != GDR_OK) return s;
    if ((s = check_ptr(state_pool, true)) != GDR_OK) return s;
    if (slot == nullptr || reinterpret_cast<uintptr_t>(slot) % 4 != 0) return GDR_ERR_INVALID_ARG;
    int* err = nullptr;
    if (error_word(&err) != cudaSuccess) return GDR_ERR_CUDA;
    cudaError_t e = gdr::launch_decode(*d, q, k, v, a, b, w, state_pool, o, slot, n_slots, err,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

size_t gdr_backward_workspace_size(const gdr_desc* d) {
    if (check_desc(d) != GDR_OK) return 0;
    return gdr::backward_workspace_bytes(*d, 0);
}

size_t gdr_backward_varlen_workspace_size(const gdr_desc* d, int n_seqs) {
    if (check_desc(d) != GDR_OK || n_seqs < 1) return 0;
    return gdr::backward_workspace_bytes(*d, n_seqs);
}

namespace {
gdr_status backward_impl(const gdr_desc* d, const int* cu_seqlens, int n_seqs, const void* q,
                         const void* k, const void* v, const void* a, const void* b,
                         const void* w, const float* s0, const void* d_o,
                         const float* ds_final, void* dq, void* dk, void* dv, void* da,
                         void* db, void* dw, float* ds0, void* workspace, size_t ws_bytes,
                         gdr_stream_t stream) {
    gdr_status s = check_desc(d);
    if (s != GDR_OK) return s;
    const bool have_tokens = d->T > 0;
    if ((s = check_inputs(d, have_tokens, q, k, v, a, b, w, d_o)) != GDR_OK) return s;
    if ((s = check_inputs(d, have_tokens, dq, dk, dv, da, db, dw, d_o)) != GDR_OK) return s;
    if ((s = check_ptr(s0, false)) != GDR_OK) return s;
    if ((s = check_ptr(ds_final, false)) != GDR_OK) return s;
    if ((s = check_ptr(ds0, false)) != GDR_OK) return s;
    const size_t need = gdr::backward_workspace_bytes(*d, cu_seqlens ? n_seqs : 0);
    if (workspace == nullptr || ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDR_ERR_INVALID_ARG;
    if (ds0 == nullptr && !have_tokens) return GDR_OK;  // nothing to write

    int* err = nullptr;
    if (error_word(&err) != cudaSuccess) return GDR_ERR_CUDA;
    const void* in[6] = {q, k, v, a, b, w};
    void* grads[6] = {dq, dk, dv, da, db, dw};
    cudaError_t e = gdr::launch_backward(*d, cu_seqlens, n_seqs, in, s0, d_o, ds_final, grads,
                                         ds0, workspace, err,
                                         reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}
}  // namespace

gdr_status gdr_backward_chunked(const gdr_desc* d, const void* q, const void* k, const void* v,
                                const void* a, const void* b, const void* w, const float* s0,
                                const void* d_o, const float* ds_final, void* dq, void* dk,
                                void* dv, void* da, void* db, void* dw, float* ds0,
                                void* workspace, size_t ws_bytes, gdr_stream_t stream) {
    return backward_impl(d, nullptr, 0, q, k, v, a, b, w, s0, d_o, ds_final, dq, dk, dv, da, db,
                         dw, ds0, workspace, ws_bytes, stream);
}

gdr_status gdr_backward_varlen(const gdr_desc* d, const int* cu_seqlens, int n_seqs,
                               const void* q, const void* k, const void* v, const void* a,
                               const void* b, const void* w, const float* s0, const void* d_o,
                               const float* ds_final, void* dq, void* dk, void* dv, void* da,
                               void* db, void* dw, float* ds0, void* workspace,
                               size_t ws_bytes, gdr_stream_t stream) {
    if (!d || d->B != 1 || n_seqs < 1) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr || reinterpret_cast<uintptr_t>(cu_seqlens) % 4 != 0)
        return GDR_ERR_INVALID_ARG;
    if ((long long)n_seqs * d->H > 0x7fffffffLL) return GDR_ERR_INVALID_ARG;
    return backward_impl(d, cu_seqlens, n_seqs, q, k, v, a, b, w, s0, d_o, ds_final, dq, dk, dv,
                         da, db, dw, ds0, workspace, ws_bytes, stream);
}

// ---- backward with library-owned scratch (gdr_backward_chunked_noalloc)
//
// Some callers cannot allocate device memory at all: a plugin running inside
// a host runtime that owns every byte of device memory and hands the library
// no allocator, or code on a latency-critical path where cudaMalloc is ruled
// out because it may synchronise the device.  For them the backward pass can
// use this file-scope scratch instead of a caller-supplied workspace.  It is
// a __device__ array: every GPU on which the library's module is loaded holds
// GDR_NOALLOC_SCRATCH_BYTES of it until the process exits, and all calls on
// that GPU share it.
} // extern "C"
static __device__ __align__(256) unsigned char g_gdr_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];  // device address of the scratch, per device (g_mu)

// The scratch's device address on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current, and cached.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gdr_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}
}  // namespace

extern "C" {

gdr_status gdr_backward_chunked_noalloc(const gdr_desc* d, const void* q, const void* k,
                                        const void* v, const void* a, const void* b,
                                        const void* w, const float* s0, const void* d_o,
                                        const float* ds_final, void* dq, void* dk, void* dv,
                                        void* da, void* db, void* dw, float* ds0,
                                        gdr_stream_t stream) {
    gdr_status s = check_desc(d);
    if (s != GDR_OK) return s;
    // larger than the scratch: refused before any CUDA call
    if (gdr::backward_workspace_bytes(*d, 0) > (size_t)GDR_NOALLOC_SCRATCH_BYTES)
        return GDR_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    // The backward writes every word of its workspace before it reads it
    // (chunk-start states from s0, the running dS from ds_final), so nothing
    // left in the scratch by an earlier call needs clearing.
    return backward_impl(d, nullptr, 0, q, k, v, a, b, w, s0, d_o, ds_final, dq, dk, dv, da, db,
                         dw, ds0, scratch, (size_t)GDR_NOALLOC_SCRATCH_BYTES, stream);
}

void gdr_test_skip_signal(int enable) { g_test_skip_signal.store(enable ? 1 : 0); }

gdr_status gdr_last_device_error(gdr_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDR_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_gdr_error_word, sizeof(int)) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (word == 0) return GDR_OK;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_gdr_error_word, &zero, sizeof(int)) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (word & gdr::kErrTimeout) return GDR_ERR_TIMEOUT;
    if (word & gdr::kErrIndex) return GDR_ERR_INVALID_ARG;
    return GDR_ERR_RANGE;
}

}  // extern "C"
