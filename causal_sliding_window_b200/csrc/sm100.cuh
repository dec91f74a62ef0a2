// sm100.cuh -- thin inline-PTX layer for sm_100a: mbarriers, TMA tile loads,
// tcgen05 MMA / TMEM, and bounded waits.
//
// Everything here is a direct wrapper over one PTX instruction (PTX ISA 8.7+,
// "tcgen05" and "cp.async.bulk.tensor" sections).  Descriptor bit layouts
// follow the sm_100 UMMA shared-memory and instruction descriptor formats.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace swa {

// ---------------------------------------------------------------------------
// Status words.  A wait that gives up (see mbar_wait), or a data-dependent error
// (cache overflow, position outside the rotary tables), ORs a code into the
// device-wide word g_attn_status (read by attn_device_status) and into the word
// of the stream slot the launch was given (read by attn_poll_device_status).
// The host maps each (device, stream) pair to one of kStreamSlots slots; the
// same index names the launch's work counter (g_work_slots below).
// ---------------------------------------------------------------------------
constexpr int kStreamSlots = 64;
__device__ int g_attn_status;
__device__ int g_stream_status[kStreamSlots];

enum : int {
    kStatusTimeoutProducer = 1,
    kStatusTimeoutMma = 2,
    kStatusTimeoutSoftmax = 4,
    kStatusTimeoutEpilogue = 8,
    kStatusTimeoutSelftest = 16,
    kStatusSmemLayout = 32,   // dynamic shared memory too misaligned for the tile layout
    kStatusCacheOverflow = 64,   // a prefill chunk did not fit in the cache capacity
    kStatusPositionRange = 128,  // a token position outside the rotary tables
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void report_status(int slot, int code) {
    atomicOr(&g_attn_status, code);
    atomicOr(&g_stream_status[slot & (kStreamSlots - 1)], code);
}

__device__ __forceinline__ long long imax_ll(long long a, long long b) { return a > b ? a : b; }
__device__ __forceinline__ long long imin_ll(long long a, long long b) { return a < b ? a : b; }

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Gives up after
// `limit_cycles` SM clocks, or as soon as another role of the CTA has given up
// (shared `abort_flag[0]`).  On giving up it records `code` in the status words
// (abort_flag[1] holds the launch's stream slot) and returns false; callers then
// stop issuing work and fall through to the kernel's teardown.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit_cycles, int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (abort_flag[0]) return false;
        if (clock64() - t0 > limit_cycles) {
            abort_flag[0] = 1;
            report_status(abort_flag[1], code);
            return false;
        }
    }
}

// Bounded wait used before a CTA exits, for copies it issued itself: unlike mbar_wait it
// keeps waiting after another role has given up (a TMA copy that was issued completes on
// its own), but still stops after `limit_cycles`.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, long long limit_cycles, int slot) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit_cycles) {
            report_status(slot, kStatusTimeoutProducer);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// Dynamic work distribution for persistent kernels.
//
// A launch of a persistent kernel draws item indices 0, 1, 2, ... from one counter in
// g_work_slots (atomicAdd), so whichever CTA is free takes the next item: items keep the
// kernel's order (head-major, heaviest first) and the load balances itself.  Inside a CTA
// the producer thread draws the index and hands it to the other roles through a small
// shared-memory ring (item_full / item_empty mbarriers).  When a CTA stops drawing it
// counts itself done; the last CTA of the launch zeroes the slot for a later launch.  The
// slot is the launch's stream slot: launches on one stream run one after another, so they
// can share it, and launches on streams with different slots never touch each other's.
// ---------------------------------------------------------------------------
constexpr int kWorkSlots = kStreamSlots;
constexpr int kItemRing = 4;
struct WorkSlot {
    int next;
    int done;
};
__device__ WorkSlot g_work_slots[kWorkSlots];

// Producer side: draw the k-th item of this CTA and publish it in ring entry k % kItemRing.
__device__ __forceinline__ int item_produce(int slot, int k, volatile int* ring, uint32_t full0, uint32_t empty0,
                                            volatile int* abort_flag, long long limit, bool& ok) {
    const int e = k % kItemRing;
    if (k >= kItemRing)
        ok = ok && mbar_wait(empty0 + 8u * e, uint32_t(((k / kItemRing) - 1) & 1), abort_flag, limit,
                             kStatusTimeoutProducer);
    const int item = ok ? atomicAdd(&g_work_slots[slot].next, 1) : 0x7fffffff;
    ring[e] = item;
    mbar_arrive(full0 + 8u * e);
    return item;
}

// Consumer side (every lane of a consuming warp calls it; lane 0 releases the entry).
__device__ __forceinline__ int item_consume_warp(int k, volatile int* ring, uint32_t full0, uint32_t empty0,
                                                 volatile int* abort_flag, long long limit, int code, bool& ok) {
    const int e = k % kItemRing;
    ok = ok && __all_sync(0xffffffffu, mbar_wait(full0 + 8u * e, uint32_t((k / kItemRing) & 1), abort_flag,
                                                 limit, code));
    const int item = ok ? ring[e] : 0x7fffffff;
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(empty0 + 8u * e);
    return item;
}

// Consumer side for a single thread (one arrival).
__device__ __forceinline__ int item_consume_thread(int k, volatile int* ring, uint32_t full0, uint32_t empty0,
                                                   volatile int* abort_flag, long long limit, int code, bool& ok) {
    const int e = k % kItemRing;
    ok = ok && mbar_wait(full0 + 8u * e, uint32_t((k / kItemRing) & 1), abort_flag, limit, code);
    const int item = ok ? ring[e] : 0x7fffffff;
    mbar_arrive(empty0 + 8u * e);
    return item;
}

// Called once per CTA by the producer thread after its last draw.
__device__ __forceinline__ void work_slot_finish(int slot) {
    __threadfence();
    if (atomicAdd(&g_work_slots[slot].done, 1) == int(gridDim.x) - 1) {
        g_work_slots[slot].next = 0;
        g_work_slots[slot].done = 0;
        __threadfence();
    }
}

// ---------------------------------------------------------------------------
// TMA: 4-D tiled load global -> shared, completion counted on an mbarrier.
// Coordinates are innermost first.  (No cluster multicast anywhere.)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Hint: bring one tile of a tensor map into L2 (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// 4-D tiled store shared -> global (bulk-group completion); rows outside the tensor are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group of this thread has finished reading its shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Barrier over `nthreads` threads (whole warps) on named barrier `id` (1..15).
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Untiled bulk copy global -> shared (both 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, fences, commit, MMA, TMEM load/store.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T   (kind::f16, fp32 accumulate)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
//   [4,6) D format (1 = f32)   [7,10) A format (1 = bf16)   [10,13) B format (1 = bf16)
//   [15] A major (0 = K, 1 = MN)   [16] B major   [17,23) N >> 3   [24,29) M >> 4
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   [0,14) start address >> 4   [16,30) leading byte offset >> 4
//   [32,46) stride byte offset >> 4   [46,48) version (1 on sm_100)   [61,64) layout (2 = SWIZZLE_128B)
// K-major tiles: rows of 128 B, 8-row groups `sbo` apart (lbo unused, 16).
// MN-major tiles: 64-element MN chunks `lbo` apart, 8-row K groups `sbo` apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

// The same descriptor split into its two 32-bit words, for the issue loops: lo holds the start
// address (>> 4, bits 0..13) and the leading byte offset (bits 16..29), hi the stride byte offset,
// the version and the swizzle mode.  An operand n bytes further on is lo + (n >> 4) (shared-memory
// addresses stay below 2^18, so the 14-bit address field never carries), which keeps the issuing
// thread to one integer add per operand and MMA.
struct SDesc {
    uint32_t lo, hi;
};
__device__ __forceinline__ SDesc sdesc_sw128_w(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return {((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16), ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29)};
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T (kind::f16), descriptors as (lo, hi) words.
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint32_t alo, uint32_t ahi, uint32_t blo, uint32_t bhi,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "mov.b64 da, {%1, %2};\n\t"
        "mov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}\n" ::"r"(d_tmem),
        "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T (kind::f16), B as (lo, hi) words.
__device__ __forceinline__ void mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t blo, uint32_t bhi,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM words: thread i of the warp gets
// columns [c, c+32) of lane (warp quarter * 32 + i).
#define SWA_R8(o) "=r"(r[o + 0]), "=r"(r[o + 1]), "=r"(r[o + 2]), "=r"(r[o + 3]), "=r"(r[o + 4]), \
                  "=r"(r[o + 5]), "=r"(r[o + 6]), "=r"(r[o + 7])
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : SWA_R8(0), SWA_R8(8), SWA_R8(16), SWA_R8(24)
        : "r"(taddr));
}
#undef SWA_R8

// Wait for this thread's outstanding tcgen05.ld; the "+r" operands pin every
// use of the loaded registers after the wait.
#define SWA_W8(o) "+r"(r[o + 0]), "+r"(r[o + 1]), "+r"(r[o + 2]), "+r"(r[o + 3]), "+r"(r[o + 4]), \
                  "+r"(r[o + 5]), "+r"(r[o + 6]), "+r"(r[o + 7])
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : SWA_W8(0), SWA_W8(8), SWA_W8(16), SWA_W8(24)::"memory");
}
#undef SWA_W8

// 32 lanes x 16 columns.
#define SWA_R8(o) "=r"(r[o + 0]), "=r"(r[o + 1]), "=r"(r[o + 2]), "=r"(r[o + 3]), "=r"(r[o + 4]), \
                  "=r"(r[o + 5]), "=r"(r[o + 6]), "=r"(r[o + 7])
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : SWA_R8(0), SWA_R8(8)
        : "r"(taddr));
}
#undef SWA_R8
#define SWA_W8(o) "+r"(r[o + 0]), "+r"(r[o + 1]), "+r"(r[o + 2]), "+r"(r[o + 3]), "+r"(r[o + 4]), \
                  "+r"(r[o + 5]), "+r"(r[o + 6]), "+r"(r[o + 7])
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : SWA_W8(0), SWA_W8(8)::"memory");
}
#undef SWA_W8

#define SWA_S8(o) "r"(r[o + 0]), "r"(r[o + 1]), "r"(r[o + 2]), "r"(r[o + 3]), "r"(r[o + 4]), "r"(r[o + 5]), \
                  "r"(r[o + 6]), "r"(r[o + 7])
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        SWA_S8(0), SWA_S8(8), SWA_S8(16), SWA_S8(24)
        : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        SWA_S8(0), SWA_S8(8)
        : "memory");
}
#undef SWA_S8
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory vector load by shared-window address (always the LDS path).
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------------------
// Small math helpers (single PTX instructions).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Pack two fp32 into bf16x2 with round-to-nearest-even; `lo` lands in bits [0,16).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One 32-byte global store (a whole sector); ptr must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

// N fp32 values v[0..N) times mul, as bf16 at dst (N a multiple of 16): 32-byte stores when dst is
// 32-byte aligned, else 16-byte ones (dst is always 16-byte aligned).  A thread writing its own
// row this way issues half the store instructions of 16-byte stores.
template <int N>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float* v, float mul) {
    if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[16 * k + 2 * i] * mul, v[16 * k + 2 * i + 1] * mul);
            st_global_v8(dst + 16 * k, w);
        }
    } else {
#pragma unroll
        for (int k = 0; k < N / 8; ++k) {
            uint4 w;
            w.x = pack_bf16x2(v[8 * k + 0] * mul, v[8 * k + 1] * mul);
            w.y = pack_bf16x2(v[8 * k + 2] * mul, v[8 * k + 3] * mul);
            w.z = pack_bf16x2(v[8 * k + 4] * mul, v[8 * k + 5] * mul);
            w.w = pack_bf16x2(v[8 * k + 6] * mul, v[8 * k + 7] * mul);
            *reinterpret_cast<uint4*>(dst + 8 * k) = w;
        }
    }
}
// Same packing on the integer pipe, for finite inputs: add half a bf16 ulp to the magnitude
// bits and keep the high halves (round to nearest, ties away from zero; differs from
// pack_bf16x2 only on exact ties).  Two adds and one byte permute, so the conversions of
// a score tile do not compete with exp2 for the special-function unit.
__device__ __forceinline__ uint32_t pack_bf16x2_alu(float lo, float hi) {
    const uint32_t a = __float_as_uint(lo) + 0x8000u, b = __float_as_uint(hi) + 0x8000u;
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

}  // namespace swa
