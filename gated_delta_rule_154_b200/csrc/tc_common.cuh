// tc_common.cuh -- Blackwell (sm_100a) tensor-core building blocks written
// directly in PTX: shared-memory matrix descriptors, tcgen05.mma (kind::f16,
// bf16 operands, float32 accumulation in tensor memory), tcgen05.commit to an
// mbarrier, bounded mbarrier waits, tensor-memory allocation and 32x32b
// loads/stores.
//
// Operand tiles live in shared memory in one "row-major, 128-byte swizzled"
// format: a tile of R rows and 64*P bf16 columns is stored as P panels of
// R rows x 128 bytes (panel p holds columns 64p .. 64p+63); inside a panel,
// row r starts at r*128 and its eight 16-byte chunks are permuted by
// chunk ^ (r % 8).  Every panel starts on a 1024-byte boundary.  The same
// bytes describe
//   * a K-major operand whose M (or N) index is the row and K the column, and
//   * an MN-major operand whose K index is the row and M (or N) the column,
// so a [token][channel] tile feeds both kinds of product without a copy.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gdr {
namespace tc {

// ------------------------------------------------------------ smem addresses

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (row, col) inside a swizzled tile whose panels are
// `panel_bytes` apart.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, uint32_t panel_bytes) {
    const int p = col >> 6, c = col & 63;
    return (uint32_t)p * panel_bytes + (uint32_t)row * 128u +
           ((uint32_t)(((c >> 3) ^ (row & 7))) << 4) + ((uint32_t)(c & 7) << 1);
}

// Pack two floats into a bf16x2 word (low half = first argument).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Write one 64-column panel row (64 floats -> 64 bf16 = 128 bytes) of a
// swizzled tile with eight 16-byte stores.  `row_base` points at the panel.
__device__ __forceinline__ void store_row64_bf16(uint8_t* panel_base, int row, const float* v) {
    uint8_t* rp = panel_base + row * 128;
#pragma unroll
    for (int c16 = 0; c16 < 8; ++c16) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * c16 + 0], v[8 * c16 + 1]);
        w.y = pack_bf16x2(v[8 * c16 + 2], v[8 * c16 + 3]);
        w.z = pack_bf16x2(v[8 * c16 + 4], v[8 * c16 + 5]);
        w.w = pack_bf16x2(v[8 * c16 + 6], v[8 * c16 + 7]);
        *reinterpret_cast<uint4*>(rp + ((c16 ^ (row & 7)) << 4)) = w;
    }
}

// Same for 32 columns starting at column 32*half of the panel (16-byte chunks
// 4*half .. 4*half+3).
__device__ __forceinline__ void store_row32_bf16(uint8_t* panel_base, int row, int half,
                                                 const float* v) {
    uint8_t* rp = panel_base + row * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c16 = 4 * half + q;
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4*>(rp + ((c16 ^ (row & 7)) << 4)) = w;
    }
}

// Same for 16 columns starting at column 16*q of the panel (16-byte chunks
// 2q, 2q+1).
__device__ __forceinline__ void store_row16_bf16(uint8_t* panel_base, int row, int q,
                                                 const float* v) {
    uint8_t* rp = panel_base + row * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c16 = 2 * q + h;
        uint4 w;
        w.x = pack_bf16x2(v[8 * h + 0], v[8 * h + 1]);
        w.y = pack_bf16x2(v[8 * h + 2], v[8 * h + 3]);
        w.z = pack_bf16x2(v[8 * h + 4], v[8 * h + 5]);
        w.w = pack_bf16x2(v[8 * h + 6], v[8 * h + 7]);
        *reinterpret_cast<uint4*>(rp + ((c16 ^ (row & 7)) << 4)) = w;
    }
}

// ------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor (tcgen05 form): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;   // version
    d |= (uint64_t)2u << 61;   // SWIZZLE_128B
    return d;
}

// K-major operand: rows are M (or N), columns are K.  K step kk covers
// columns 16kk .. 16kk+15: panel kk/4, byte offset 32*(kk%4) in the row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, uint32_t panel_bytes, int kk) {
    return make_desc(tile_saddr + (uint32_t)(kk >> 2) * panel_bytes + (uint32_t)(kk & 3) * 32u,
                     16u, 1024u);
}

// MN-major operand: rows are K, columns are M (or N).  K step kk covers rows
// 16kk .. 16kk+15 (two 8-row groups, 1024 bytes apart); panels hold 64
// consecutive M (or N) indices, `panel_bytes` apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile_saddr, uint32_t panel_bytes, int kk) {
    return make_desc(tile_saddr + (uint32_t)kk * 2048u, panel_bytes, 1024u);
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, float32 D,
// shape M x N, operand majors (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((uint32_t)a_mn << 15)           // A major
           | ((uint32_t)b_mn << 16)           // B major
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// ------------------------------------------------------------- tcgen05 ops

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
}

// Same with A read from tensor memory: M rows in lanes, K packed two bf16 per
// 32-bit column (the lower half holds the even k), one K = 16 step spanning 8
// columns from `a_tmem`.  A is K-major there.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, bool accumulate) {
    const uint32_t acc = accumulate ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc));
}

// Make `bar` track completion of every tcgen05.mma this thread issued so far.
__device__ __forceinline__ void mma_commit(uint32_t bar_saddr) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            bar_saddr)
        : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy writes to shared memory become visible to tcgen05.mma.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Allocate / free tensor memory (one full warp).  The base address is
// written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_saddr),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 lanes x 32 consecutive columns: thread i of the warp gets lane
// (lane_base + i), columns col .. col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// 32 lanes x 16 consecutive columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive columns as raw 32-bit words (e.g. packed bf16 pairs).
__device__ __forceinline__ void tmem_ld16u(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint32_t bar_saddr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_saddr), "r"(count)
                 : "memory");
}

// Make an initialised mbarrier visible to the asynchronous proxy.
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_saddr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar_saddr), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait until the barrier's phase with parity `parity` has completed, for at
// most `limit_ns` nanoseconds.  Returns false if the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar_saddr, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar_saddr, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar_saddr, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// One plain arrival (release semantics) on a barrier initialised with count 1.
__device__ __forceinline__ void mbar_arrive(uint32_t bar_saddr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_saddr) : "memory");
}

// ------------------------------------------------------------- TMA loads

// Arm `bar` for one arrival plus `bytes` of asynchronous transactions.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar_saddr, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_saddr),
                 "r"(bytes)
                 : "memory");
}

// 4-D tiled bulk-tensor load into shared memory, completion counted on `bar`
// in bytes.  Coordinates are innermost first.  (Plain load: no multicast.)
__device__ __forceinline__ void tma_load_4d(uint32_t dst_saddr, const void* tmap, int c0, int c1,
                                            int c2, int c3, uint32_t bar_saddr) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst_saddr),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(bar_saddr)
        : "memory");
}

// 4-D tiled bulk-tensor store from shared memory (bulk-group completion).
// Rows past the tensor's extent are not written.
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t src_saddr, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group "
        "[%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(src_saddr), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Bring `bytes` (a multiple of 16) of global memory at `gptr` into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* gptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                     reinterpret_cast<uint64_t>(gptr)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

}  // namespace tc
}  // namespace gdr
