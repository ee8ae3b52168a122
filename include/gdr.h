/*
 * gdr.h -- C ABI of the gated delta-rule recurrence library (libgdr.so),
 * CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * The operation.  Per (batch b, head h), with a state S in R^{dk x dv} whose
 * rows index key channels and columns index value channels, each token t does
 *
 *     S'  = Diag(a_t) S_{t-1}                          decay
 *     S_t = S' - (b_t * k_t)(k_t^T S') + k_t (w_t * v_t)^T   erase, then write
 *     o_t = S_t^T q_t                                   read-out
 *
 * Sources: the update rule and its order (decay, erase from the decayed state,
 * write) -- page "FG^2-GDN: Enhancing Long-Context Gated Delta Networks with
 * Doubly Fine-Grained Control" (gist.science 2604.19021), section 2
 * "Methodology", FG2-GDN update rule; the decoupled per-channel erase gate b_t
 * (key side) and write gate w_t (value side) with KDA's per-channel decay --
 * page "Gated DeltaNet-2: decoupling erase and write in linear attention"
 * (needhelp.icu), the gates table; scalar decay (Gated DeltaNet) versus
 * per-channel decay (KDA) -- FG^2-GDN page, section 1 "Problem statement";
 * the chunkwise-parallel (WY) evaluation used by gdr_forward_chunked --
 * FG^2-GDN page, section 2 (rank-1 Householder structure kept for WY chunked
 * training) and section 3 (DPLR structure, KDA-style chunked kernels); the
 * fixed-size state that replaces a KV cache and makes decoding O(1) in memory
 * -- Gated DeltaNet-2 page, "The attention bottleneck".  The read-out with the
 * updated state, no 1/sqrt(dk) on q, and q, k normalised by the caller are
 * readings where the pages print no equation.
 *
 * Conventions shared by every entry point.
 *   - Tensors are dense, row-major, contiguous, in device memory owned by the
 *     caller: q, k [B, T, H, dk]; v, o [B, T, H, dv]; vector gates a, b
 *     [B, T, H, dk] and w [B, T, H, dv]; scalar gates [B, T, H] (one value per
 *     token and head); states [B, H, dk, dv] in float32.
 *   - q, k, v, the gates and o share in_dtype (float32 or bf16); the state is
 *     always float32.  Arithmetic is float32 (tensor-core products take bf16
 *     operands with float32 accumulation on the bf16 path).
 *   - q and k are expected L2-normalised by the caller; a_t in (0, 1].
 *   - Every pointer the call reads or writes must be 16-byte aligned.
 *   - The library allocates nothing and keeps no per-call state.  Calls are
 *     asynchronous on `stream` (0 = the legacy default stream).
 *   - Argument errors are reported synchronously, before anything is
 *     launched; nothing is written in that case.  A failed launch returns
 *     GDR_ERR_CUDA.  Faults found on the device (a bounded wait that ran out,
 *     decay outside the supported range) are recorded in a per-device error
 *     word read by gdr_last_device_error().  No C++ exception crosses the ABI.
 *   - Concurrent calls on distinct buffers are safe.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gdr_stream_t; /* same type as cudaStream_t */

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad enum */
    GDR_ERR_UNSUPPORTED = 2, /* valid, but no kernel for this combination  */
    GDR_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
    GDR_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed        */
    GDR_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out              */
    GDR_ERR_RANGE = 6        /* device: decay too strong for the chunk form */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/* How a gate is given.  ONE: the gate is identically 1 and its pointer is
 * ignored (may be NULL).  SCALAR: one value per (b, t, h), [B, T, H].
 * VECTOR: one value per channel, [B, T, H, dk] for a and b, [B, T, H, dv]
 * for w.
 * FG2 (erase and write only): the tensor holds FG^2-GDN's per-channel
 * learning rate beta >= 0, laid out as VECTOR, and enters through its square
 * root.  erase = FG2: the key used everywhere is sqrt(beta^k) * k and the
 * erase gate is 1.  write = FG2: the write gate is sqrt(beta^v).  With both
 * FG2 and one tensor for b and w this is FG^2-GDN's symmetric update
 *     S_t = (I - k~ k~^T) Diag(a_t) S_{t-1} + k~ v~^T,  k~ = sqrt(beta) k,
 *     v~ = sqrt(beta) v
 * (FG^2-GDN page, section 2 "Methodology", FG2-GDN update rule); with
 * separate beta^k and beta^v tensors it is the reading taken for FG^2-GDN+
 * (same page, the FG2-GDN+ variant, which prints no formula).  The square
 * roots are taken inside the kernels; no scaled copy of k, v is written. */
typedef enum {
    GDR_GATE_ONE = 0,
    GDR_GATE_SCALAR = 1,
    GDR_GATE_VECTOR = 2,
    GDR_GATE_FG2 = 3
} gdr_gate;

typedef struct {
    int B, T, H;          /* batch, tokens, heads; B, H >= 1, T >= 0        */
    int dk, dv;           /* 64 or 128 each                                 */
    int chunk;            /* chunk length of the chunked form: 16, 32 or 64 */
    gdr_dtype in_dtype;   /* dtype of q, k, v, a, b, w and o                */
    gdr_gate decay;       /* a */
    gdr_gate erase;       /* b */
    gdr_gate write;       /* w; b and w may be the same tensor (shared beta) */
} gdr_desc;

/* Bytes of device workspace gdr_forward_chunked can use for `desc` (0 if none,
 * or if desc is invalid).  Non-zero only where the call splits the sequences
 * (see gdr_forward_chunked): bf16, dk = dv = 128, chunk 64, B * H <= 37 heads
 * and T >= 4096 * P with P = 148 / (B * H).  Pure host function, no CUDA
 * call. */
size_t gdr_workspace_size(const gdr_desc *desc);

/*
 * Causal prefill over T tokens by the chunkwise-parallel form: per chunk of
 * `chunk` tokens, cumulative decay, intra-chunk gram matrices, a triangular
 * (UT-transform) solve for the erase terms, and a sequential pass over
 * chunks that carries S in float32.  Equal, up to rounding, to running the
 * recurrence above token by token.
 *
 *   q, k, v, a, b, w  inputs as described above (a/b/w ignored when ONE)
 *   s0       [B, H, dk, dv] float32 initial state, or NULL for zeros
 *   o        [B, T, H, dv] in_dtype, written
 *   s_final  [B, H, dk, dv] float32 final state, or NULL (not written);
 *            may equal s0 (in-place update)
 *   workspace, ws_bytes  device scratch of gdr_workspace_size(desc) bytes,
 *            or NULL / 0.  When gdr_workspace_size is non-zero (few heads,
 *            long sequences: most SMs would idle with one CTA per head) and
 *            the workspace is given, every sequence is split into
 *            P = 148 / (B * H) segments run side by side through
 *            gdr_forward_segmented; with NULL the one-pass kernel runs.  A
 *            non-NULL workspace smaller than required: GDR_ERR_WORKSPACE.
 *            gdr_forward_varlen takes no workspace.
 *
 * Supported: dk, dv in {64, 128}; float32 inputs with chunk in {16, 32, 64}
 * (chunk <= 32 when dk = 128); bf16 inputs with chunk 64 and dk = dv = 128 on
 * the tensor-core kernel, and the float32 kernel's chunk sizes otherwise.
 * Other valid descriptors return GDR_ERR_UNSUPPORTED.
 *
 * Decay range: within each chunk the products of a over any run of tokens
 * must stay representable in float32 after the kernel's factorisation
 * (about exp(-80) over half a chunk per channel on the bf16 tensor-core
 * kernel); outside it the device error word reports GDR_ERR_RANGE.
 */
gdr_status gdr_forward_chunked(const gdr_desc *desc, const void *q, const void *k,
                               const void *v, const void *a, const void *b,
                               const void *w, const float *s0, void *o,
                               float *s_final, void *workspace, size_t ws_bytes,
                               gdr_stream_t stream);

/*
 * The same prefill over packed sequences of different lengths (varlen):
 * desc->B must be 1 and desc->T is the total token count; q, k, v, the gates
 * and o are [1, T, H, *] with sequence n occupying tokens
 * [cu_seqlens[n], cu_seqlens[n + 1]).  cu_seqlens: int32 [n_seqs + 1] in
 * device memory, 4-byte aligned, non-decreasing, cu_seqlens[0] = 0 and
 * cu_seqlens[n_seqs] <= T; every sequence starts from its own state and no
 * token of one sequence affects another.  s0 and s_final are
 * [n_seqs, H, dk, dv] float32 (s0 may be NULL for zeros).  A sequence whose
 * range falls outside [0, T] is skipped (its o and s_final are not written)
 * and recorded in the device error word, read as GDR_ERR_INVALID_ARG by
 * gdr_last_device_error().  Everything else as gdr_forward_chunked.
 */
gdr_status gdr_forward_varlen(const gdr_desc *desc, const int *cu_seqlens, int n_seqs,
                              const void *q, const void *k, const void *v, const void *a,
                              const void *b, const void *w, const float *s0, void *o,
                              float *s_final, void *workspace, size_t ws_bytes,
                              gdr_stream_t stream);

/*
 * One decode step (desc->T must be 1): reads and rewrites `state` in place.
 * Shapes drop the T axis: q, k, a, b [B, H, dk] (scalar gates [B, H]);
 * v, w [B, H, dv]; state [B, H, dk, dv] float32; o [B, H, dv] in_dtype.
 * Each state element is read once and written once.
 */
gdr_status gdr_decode_step(const gdr_desc *desc, const void *q, const void *k,
                           const void *v, const void *a, const void *b,
                           const void *w, float *state, void *o,
                           gdr_stream_t stream);

/*
 * The same step over a pool of states (many sequences, one state pool):
 * batch entry b reads and rewrites state_pool[slot[b]], each pool slot being
 * [H, dk, dv] float32; the pool holds n_slots >= 1 of them, other slots are
 * not touched.  slot: int32 [B] in device memory, 4-byte aligned.  Entries
 * must be distinct (two entries on one slot race).  An entry outside
 * [0, n_slots) is skipped (its o is not written) and recorded in the device
 * error word, read as GDR_ERR_INVALID_ARG by gdr_last_device_error().
 * Everything else as gdr_decode_step.
 */
gdr_status gdr_decode_step_paged(const gdr_desc *desc, const void *q, const void *k,
                                 const void *v, const void *a, const void *b,
                                 const void *w, float *state_pool, const int *slot,
                                 int n_slots, void *o, gdr_stream_t stream);

/* Bytes of device workspace gdr_backward_chunked needs for `desc`; 0 if desc
 * is invalid.  Pure host function, no CUDA call.
 *   - bf16 with dk = dv = 128 and T > 0 (the tensor-core path): the scaled
 *     state at the start of every 64-token chunk (bf16) and the final state
 *     (float32), every chunk's E (bf16), five bf16 [B, T, H, 128]
 *     intermediates and two float32 rows per chunk and head:
 *     B * H * (ceil(T / 64) * 33792 + 65536) + B * T * H * 1536 bytes.
 *   - otherwise: the state at the start of every 32-token chunk plus one
 *     running state gradient, B * H * dk * dv * 4 * (ceil(T / 32) + 1). */
size_t gdr_backward_workspace_size(const gdr_desc *desc);

/*
 * Gradients of the prefill (training).  With the loss
 *     L = sum_t <o_t, do_t> + <S_T, ds_final>,
 * where o and S_T are what gdr_forward_chunked returns for the same inputs,
 * the call writes dL/dq, dL/dk, dL/dv, dL/da, dL/db, dL/dw and dL/ds0.  The
 * pages train this recurrence through its chunkwise (WY) form (FG^2-GDN
 * page, section 2 "Methodology"); the call differentiates that form: a
 * forward pass stores the state at the start of every chunk in the
 * workspace, then one CTA per (batch, head) walks the chunks backwards
 * carrying dS.
 *   - bf16 inputs with dk = dv = 128, T > 0: chunks of 64 tokens, three
 *     launches.  The tensor-core prefill kernel writes the chunk-start
 *     states, S_T and each chunk's key reads E; the reverse sweep runs every
 *     product on the tensor cores (bf16 operands, float32 accumulation, dS
 *     carried in float32); an elementwise kernel forms the gradients.
 *   - otherwise (float32 inputs, d = 64): chunks of 32 tokens, one launch;
 *     bf16 products on the tensor cores with tf32 operands, float32 inputs
 *     in float32 on the CUDA cores.
 * Equal, up to rounding, to differentiating the token-by-token recurrence.
 *
 *   q .. w, s0  the forward's inputs (s0 NULL for zeros); desc->chunk is not
 *            used (the pass picks its chunk length as above)
 *   d_o      [B, T, H, dv] in_dtype, the gradient on o
 *   ds_final [B, H, dk, dv] float32, the gradient on S_T, or NULL for zero
 *   dq, dk   [B, T, H, dk] in_dtype, written
 *   dv       [B, T, H, dv] in_dtype, written
 *   da, db, dw  in the shape and dtype of a, b, w (scalar gates: one value
 *            per token and head, the sum over channels); required when the
 *            gate is not ONE, ignored when it is.  With b and w the same
 *            tensor (shared beta) its gradient is db + dw.  With
 *            GDR_GATE_FG2 (FG^2-GDN learning rates, beta > 0) db and dw are
 *            the gradients on beta^k and beta^v, carried through the square
 *            roots the forward takes.
 *   ds0      [B, H, dk, dv] float32, or NULL (not written); may equal
 *            ds_final
 *   workspace, ws_bytes  device scratch of gdr_backward_workspace_size(desc)
 *
 * Outputs must not overlap the inputs.  Supported: dk, dv in {64, 128},
 * float32 or bf16 inputs, every gate kind.  Decay range: every channel's
 * decay, multiplied over each 32-token chunk (tensor-core path: over tokens
 * 1-31 and 32-63 of each 64-token chunk), must stay at or above exp(-80)
 * (1e-35); otherwise the device error word reports GDR_ERR_RANGE and the
 * gradients are undefined.
 */
gdr_status gdr_backward_chunked(const gdr_desc *desc, const void *q, const void *k,
                                const void *v, const void *a, const void *b,
                                const void *w, const float *s0, const void *d_o,
                                const float *ds_final, void *dq, void *dk, void *dv,
                                void *da, void *db, void *dw, float *ds0, void *workspace,
                                size_t ws_bytes, gdr_stream_t stream);

/* Bytes of device workspace gdr_backward_varlen needs for `desc` and n_seqs
 * packed sequences: H * dk * dv * 4 * (ceil(T / 32) + 2 * n_seqs); 0 if desc
 * is invalid or n_seqs < 1.  Pure host function, no CUDA call. */
size_t gdr_backward_varlen_workspace_size(const gdr_desc *desc, int n_seqs);

/*
 * The backward over packed sequences, as gdr_forward_varlen packs them:
 * desc->B must be 1, sequence n occupies tokens [cu_seqlens[n],
 * cu_seqlens[n + 1]) of the [1, T, H, *] tensors, and s0, ds_final and ds0
 * are [n_seqs, H, dk, dv].  cu_seqlens must be non-decreasing from
 * cu_seqlens[0] >= 0 with cu_seqlens[n_seqs] <= T; a sequence for which that
 * does not hold up to its own end is skipped (its gradients are not written)
 * and recorded in the device error word (GDR_ERR_INVALID_ARG from
 * gdr_last_device_error).  Gradients of tokens outside every sequence are not
 * written.  workspace: gdr_backward_varlen_workspace_size(desc, n_seqs)
 * bytes.  Everything else as gdr_backward_chunked.
 */
gdr_status gdr_backward_varlen(const gdr_desc *desc, const int *cu_seqlens, int n_seqs,
                               const void *q, const void *k, const void *v, const void *a,
                               const void *b, const void *w, const float *s0,
                               const void *d_o, const float *ds_final, void *dq, void *dk,
                               void *dv, void *da, void *db, void *dw, float *ds0,
                               void *workspace, size_t ws_bytes, gdr_stream_t stream);

/* Bytes of the library-owned scratch that gdr_backward_chunked_noalloc uses
 * (64 MiB, held on every GPU that loads the library until the process exits). */
#define GDR_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * gdr_backward_chunked for callers that cannot allocate device memory: a
 * plugin inside a host runtime that owns all device memory and gives the
 * library no allocator, or latency-critical code that must not call
 * cudaMalloc because it may synchronise the device.  The pages have no
 * counterpart to this call; it only changes where the workspace lives.
 *
 * Arguments and results are those of gdr_backward_chunked without the
 * workspace: the call uses a file-scope scratch array of the library
 * instead, GDR_NOALLOC_SCRATCH_BYTES on each GPU.  It allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *   - Size limit: when gdr_backward_workspace_size(desc) exceeds
 *     GDR_NOALLOC_SCRATCH_BYTES the call returns GDR_ERR_WORKSPACE before any
 *     CUDA call (e.g. bf16, dk = dv = 128, B * H = 1: up to about 32k tokens).
 *   - First call on a device: it looks up the scratch's device address with
 *     cudaGetSymbolAddress on the current device and caches it.  Make that
 *     first call on each device before any stream capture begins.
 *   - Every call on a device shares the one scratch and it keeps the last
 *     call's contents; the kernel writes every word it reads, so nothing has
 *     to be cleared between calls.  Calls whose work overlaps on the GPU
 *     (other streams, or other threads of the process) race on the scratch:
 *     order them, e.g. on one stream.
 */
gdr_status gdr_backward_chunked_noalloc(const gdr_desc *desc, const void *q, const void *k,
                                        const void *v, const void *a, const void *b,
                                        const void *w, const float *s0, const void *d_o,
                                        const float *ds_final, void *dq, void *dk, void *dv,
                                        void *da, void *db, void *dw, float *ds0,
                                        gdr_stream_t stream);

/*
 * Sequence-parallel prefill.  The recurrence is affine in the state: over a
 * segment of tokens the state at its end is S_out = M S_in + N, with
 * M = prod_t (I - (b_t * k_t) k_t^T) Diag(a_t) (dk x dk) and N the segment
 * run from a zero state.  Splitting a sequence into P segments, computing
 * their (M, N) side by side, chaining them in order (the only exchange) and
 * running every segment again from its start state gives the prefill of the
 * whole sequence: long-sequence scaling as on the FG^2-GDN page
 * (gist.science 2604.19021), section 4 "Experimental results" (efficiency),
 * with the update rule of its section 2.  Supported: dk = dv = 128.
 */

/* Bytes of device workspace gdr_segment_maps needs for `desc` (the segment's
 * own B, T, H); 0 if unsupported.  Pure host function. */
size_t gdr_segment_maps_workspace_size(const gdr_desc *desc);

/*
 * (M, N) of one segment for every (batch, head): desc, q .. w describe the
 * segment's tokens exactly as for gdr_forward_chunked.  m_out [B, H, dk, dk]
 * float32: the segment run from S = I with every write switched off (a
 * scalar write gate of 0); n_out [B, H, dk, dv] float32: the segment run from
 * S = 0.  Two prefill launches; their outputs o go to the workspace and are
 * discarded.  Errors as gdr_forward_chunked; GDR_ERR_UNSUPPORTED unless
 * dk = dv = 128.
 */
gdr_status gdr_segment_maps(const gdr_desc *desc, const void *q, const void *k,
                            const void *v, const void *a, const void *b, const void *w,
                            float *m_out, float *n_out, void *workspace, size_t ws_bytes,
                            gdr_stream_t stream);

/*
 * Exclusive scan of the maps of n_segments consecutive segments, per
 * (batch, head): S = s0 (NULL: zeros); for p = 0 .. n_segments - 1 in order,
 * s_start[p] = S, then S = M_p S + N_p (float32); s_final = S.  Matrix
 * (b, p, h) of m, n and s_start is at element offset
 * (b * batch_stride + p * seg_stride + h) * dk * dv: seg_stride = B * H,
 * batch_stride = H for segment-major arrays [P, B, H, ...] (as an all-gather
 * leaves them); seg_stride = H, batch_stride = P * H for [B, P, H, ...].
 * s0 and s_final are [B, H, dk, dv]; s_start and s_final may be NULL (not
 * written).  One CTA per (batch, head).  GDR_ERR_UNSUPPORTED unless
 * dk = dv = 128.
 */
gdr_status gdr_segment_scan(int n_segments, int B, int H, int dk, int dv, long long seg_stride,
                            long long batch_stride, const float *m, const float *n,
                            const float *s0, float *s_start, float *s_final,
                            gdr_stream_t stream);

/* Bytes of device workspace gdr_forward_segmented needs; 0 if unsupported or
 * n_segments < 1.  Pure host function. */
size_t gdr_segmented_workspace_size(const gdr_desc *desc, int n_segments);

/*
 * The prefill of gdr_forward_chunked on one GPU with every sequence split into
 * n_segments segments of ceil(T / n_segments) tokens rounded up to a multiple
 * of 64 (the last ones shorter or empty).  The B x n_segments segments run as
 * packed sequences side by side: their maps (two launches), the scan, then a
 * second pass from every segment's start state that writes o.  Same
 * arguments and results as gdr_forward_chunked (o is also used as scratch by
 * the first two launches), plus a workspace of
 * gdr_segmented_workspace_size(desc, n_segments) bytes.  n_segments = 1 is
 * gdr_forward_chunked itself.
 */
gdr_status gdr_forward_segmented(const gdr_desc *desc, int n_segments, const void *q,
                                 const void *k, const void *v, const void *a, const void *b,
                                 const void *w, const float *s0, void *o, float *s_final,
                                 void *workspace, size_t ws_bytes, gdr_stream_t stream);

/* Synchronises `stream`, returns the status recorded on the device since the
 * previous call (GDR_OK if none) and clears it: GDR_ERR_TIMEOUT (a bounded
 * wait ran out), GDR_ERR_INVALID_ARG (a paged decode slot or a packed
 * sequence range out of bounds, or unordered packed sequences in the
 * backward) or
 * GDR_ERR_RANGE (decay range), in that order of precedence.  GDR_ERR_CUDA if
 * the synchronisation itself failed. */
gdr_status gdr_last_device_error(gdr_stream_t stream);

/*
 * Test hook for the bounded-wait path (fault injection without a fault).
 * After gdr_test_skip_signal(1), the next launch of the bf16 tensor-core
 * prefill leaves out the completion signal of its first chunk's gram
 * product, a signal that nothing else will set: the compute threads' wait
 * on it runs out after its limit (about 2 s), the kernel drains every copy
 * and product it has in flight, frees its tensor memory and returns, and
 * gdr_last_device_error() reports GDR_ERR_TIMEOUT.  The outputs of that
 * launch are undefined.  The request is consumed by that launch (or cleared
 * by gdr_test_skip_signal(0)); no other path reads it.  Host-only, no CUDA
 * call.
 */
void gdr_test_skip_signal(int enable);

/* Static, human-readable name of a status. */
const char *gdr_status_string(gdr_status status);

/* Library version, e.g. 0x000100 for 0.1.0. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
