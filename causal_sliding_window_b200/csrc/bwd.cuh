// bwd.cuh -- backward kernels of causal sliding-window attention.
//
// Gradients of sum(dO * O) for the forward in fwd.cuh (training runs through
// flash_attn_func, apidog guide "Train your own ChatGPT", section 5).  With
// P = softmax of the banded scores, Delta_i = sum_d dO_id O_id:
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - Delta),
//   dK = scale * dS^T Q,   dQ = scale * dS K.
//
// Three launches:
//   swa_bwd_pre_kernel      Delta and lse*log2(e) as fp32 rows [B*H, Tp] padded to
//                           Tp = 128*ceil(T/128) (padding: Delta 0, lse +inf), and a
//                           zeroed fp32 dQ accumulator
//   swa_bwd_kernel          persistent (one CTA per SM) drawing items = 128-row key/value
//                           tile of one (b, h) from a launch-wide counter (head-major,
//                           lowest key tiles first), walking the
//                           query tiles of each item's band; P^T is recomputed from lse,
//                           dK and dV stay in TMEM, and each dQ partial tile is
//                           staged in shared memory (in the Q/dO stage it was
//                           computed from) and added to the fp32 accumulator by a
//                           TMA tensor reduce-add
//   swa_bwd_dq_kernel       dQ = bf16(scale * accumulator)
//
// swa_bwd_kernel roles:
//   warp 8       TMA producer: K, V once; Q_i and dO_i per query tile into a ring
//   warp 9       MMA issuer: S^T = K Q^T, dP^T = V dO^T, dV += P^T dO (P^T from TMEM),
//                dK += dS^T Q, dQ_i = dS K
//   warps 0..3   thread = key row: P^T = exp2(S^T*scale*log2e - lse*log2e) with the
//                band mask, dS^T = P^T (dP^T - Delta) to shared memory
//   warps 4..7   thread = query row: drain dQ_i from TMEM into shared memory; one
//                thread issues the TMA reduce-add and, once it has read the tile,
//                hands the stage back to the producer
//   warps 0..7   per-item epilogue: dV (warps 0..3) and scale*dK (warps 4..7) to bf16,
//                overlapping the next item's first steps (acc_full / acc_free barriers)
#pragma once

#include "sm100.cuh"

namespace swa {

template <int D>
struct BwdCfg {
    static constexpr int BN = 128;                 // key rows per CTA (MMA M for S^T, dP^T, dV, dK)
    static constexpr int BM = 128;                 // query rows per step
    static constexpr int TILE = 128 * D * 2;
    static constexpr int BOX = 128 * 64 * 2;
    static constexpr int NBOX = D / 64;
    static constexpr int NSTAGE = 2;               // Q_i / dO_i ring
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = TILE;
    static constexpr int OFF_QD = 2 * TILE;        // stage s: Q at OFF_QD + s*2*TILE, dO after it
    static constexpr int OFF_DS = OFF_QD + NSTAGE * 2 * TILE;   // dS^T: 128 key rows x 128 query cols bf16
    static constexpr int OFF_LSE = OFF_DS + 128 * 128 * 2;      // per stage: 128 floats lse*log2e, 128 Delta
    static constexpr int OFF_BAR = OFF_LSE + NSTAGE * 2 * 128 * 4;
    // kv_full, kv_empty, qd_full x2, qd_empty x2, s_full, dp_full, p_full, ds_full, dv_done, dq_full,
    // dq_free, ds_free, mma_done, dq_staged, acc_full, acc_free; item_full, item_empty per ring entry
    static constexpr int NUM_BAR = 2 + 2 * NSTAGE + 12 + 2 * kItemRing;
    static constexpr int DQ_BOX = 128 * 32 * 4;    // one reduce box: 128 query rows x 32 fp32 columns
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    // Up to 1 KB of slack to align the tile region to 1024 bytes, within the per-block limit;
    // the kernel checks at run time that the aligned layout fits what it was given.
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;     // S^T | dP^T (then dQ) | dV | dK
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BM, 0, 0);       // K-major A, K-major B
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);      // K-major A, MN-major B
    static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 1, 1);       // MN-major A, MN-major B
    static_assert(SMEM_USED <= 232448, "shared memory");
};

struct BwdParams {
    const float* lse2;    // [B*H, Tp] lse * log2(e), +inf past T
    const float* delta;   // [B*H, Tp], 0 past T
    float* dq_acc;        // [B,T,H,D]
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    int B, T, H;
    long long W;
    float scale;
    float scale_log2;
    int n_kblk;
    int n_items;          // n_kblk * B * H
    int work_slot;        // index into g_work_slots for this launch
    int Tp;               // T rounded up to 128
    long long wait_limit;
};

// Geometry of one work item: key block kblk of head (b, h).  Items are head-major (all key
// blocks of one head, lowest first, then the next head), so the CTAs that run at the same
// time read the same head's Q / dO tiles and share them through L2.
struct BwdItem {
    int b, h, bh;
    long long k0;         // first key row
    int ilo, nsteps;      // first query tile and number of query tiles in the band
};

__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p, int item) {
    BwdItem it;
    const int kblk = item % p.n_kblk;
    it.bh = item / p.n_kblk;
    it.b = it.bh / p.H;
    it.h = it.bh % p.H;
    it.k0 = (long long)kblk * 128;
    it.ilo = int(it.k0 / 128);
    const int ihi = int(imin_ll(p.T - 1, it.k0 + 127 + p.W - 1) / 128);
    it.nsteps = ihi - it.ilo + 1;
    return it;
}

// ---------------------------------------------------------------------------
// Delta_i = sum_d dO_id * O_id and zeroing of the dQ accumulator.
// One thread per 8 consecutive elements (16 bytes) of a [B,T,H,D] row.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) swa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                          const __nv_bfloat16* __restrict__ dout,
                                                          const float* __restrict__ lse,
                                                          float* __restrict__ lse2, float* __restrict__ delta,
                                                          float* __restrict__ dq_acc, int B, int T, int H, int Tp) {
    constexpr int LPR = D / 8;   // lanes per row
    const long long nrows = (long long)B * T * H;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // lse * log2(e) into the padded rows; padding columns get +inf (and Delta 0).
    for (long long e = tid; e < (long long)B * H * Tp; e += stride) {
        const long long bh = e / Tp, t = e % Tp;
        if (t < T) {
            lse2[e] = lse[bh * T + t] * 1.4426950408889634f;
        } else {
            lse2[e] = INFINITY;
            delta[e] = 0.f;
        }
    }
    // Trip count is uniform across each group of LPR lanes (rows are LPR-aligned).
    for (long long e = tid; e < ((nrows * LPR + 31) / 32) * 32; e += stride) {
        const long long row = e / LPR;
        const int c = int(e % LPR);
        float acc = 0.f;
        if (row < nrows) {
            const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + c * 8);
            const uint4 g = *reinterpret_cast<const uint4*>(dout + row * D + c * 8);
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 fa = __bfloat1622float2(a2[i]);
                const float2 fg = __bfloat1622float2(g2[i]);
                acc = fmaf(fa.x, fg.x, acc);
                acc = fmaf(fa.y, fg.y, acc);
            }
            float4* z = reinterpret_cast<float4*>(dq_acc + row * D + c * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (row < nrows && c == 0) {
            const long long h = row % H;
            const long long bt = row / H;
            const long long t = bt % T, b = bt / T;
            delta[(b * H + h) * Tp + t] = acc;
        }
    }
}

// dq = bf16(scale * dq_acc), 8 elements per thread.
__global__ void __launch_bounds__(256) swa_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                         __nv_bfloat16* __restrict__ dq, long long n8,
                                                         float scale) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n8; e += stride) {
        const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * e];
        const float4 b = reinterpret_cast<const float4*>(dq_acc)[2 * e + 1];
        uint4 w;
        w.x = pack_bf16x2(a.x * scale, a.y * scale);
        w.y = pack_bf16x2(a.z * scale, a.w * scale);
        w.z = pack_bf16x2(b.x * scale, b.y * scale);
        w.w = pack_bf16x2(b.z * scale, b.w * scale);
        reinterpret_cast<uint4*>(dq)[e] = w;
    }
}

template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
swa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) atomicOr(&g_attn_status, kStatusSmemLayout);
        return;
    }

    const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sQD = base + C::OFF_QD, sDS = base + C::OFF_DS;
    const uint32_t sLSE = base + C::OFF_LSE;   // stage s: lse2 at sLSE + s*1024, Delta 512 bytes later
    const uint32_t bar0 = base + C::OFF_BAR;
    const uint32_t kv_full = bar0, kv_empty = bar0 + 8;
    auto qd_full = [&](int s) { return bar0 + 8u * (2 + s); };
    auto qd_empty = [&](int s) { return bar0 + 8u * (2 + C::NSTAGE + s); };
    const uint32_t bb = bar0 + 8u * (2 + 2 * C::NSTAGE);
    const uint32_t s_full = bb, dp_full = bb + 8, p_full = bb + 16, ds_full = bb + 24, dv_done = bb + 32,
                   dq_full = bb + 40, dq_free = bb + 48, ds_free = bb + 56, mma_done = bb + 64,
                   dq_staged = bb + 72, acc_full = bb + 80, acc_free = bb + 88;
    const uint32_t item_full0 = bb + 96, item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);

    const int T = p.T;
    const long long W = p.W;
    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_empty, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(qd_full(s), 1);
            mbar_init(qd_empty(s), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full, 128);
        mbar_init(ds_full, 128);
        mbar_init(dv_done, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 128);
        mbar_init(ds_free, 1);
        mbar_init(mma_done, 1);
        mbar_init(dq_staged, 128);
        mbar_init(acc_full, 1);
        mbar_init(acc_free, 256);
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 1 + 8);   // the MMA thread and warps 0..7
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tDP = tmem + 128u, tDV = tmem + 256u, tDK = tmem + 256u + uint32_t(D);

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            int n = 0, ki = 0;   // query-tile steps and items issued so far
            bool ok = true;
            for (;; ++ki) {
                const int item =
                    item_produce(p.work_slot, ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const BwdItem g = bwd_item(p, item);
                // K/V of the previous item are free once its last MMA completed.
                if (ki > 0) {
                    ok = mbar_wait(kv_empty, uint32_t((ki - 1) & 1), abort_flag, p.wait_limit, kStatusTimeoutProducer);
                    if (!ok) break;
                }
                mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
                for (int x = 0; x < C::NBOX; ++x) {
                    tma_load_4d(sK + x * C::BOX, &tm_k, kv_full, x * 64, g.h, int(g.k0), g.b);
                    tma_load_4d(sV + x * C::BOX, &tm_v, kv_full, x * 64, g.h, int(g.k0), g.b);
                }
                for (int l = 0; l < g.nsteps; ++l, ++n) {
                    const int s = n % C::NSTAGE;
                    if (!(ok = mbar_wait(qd_empty(s), ((n / C::NSTAGE) & 1) ^ 1u, abort_flag, p.wait_limit,
                                         kStatusTimeoutProducer)))
                        break;
                    const int qrow = (g.ilo + l) * C::BM;
                    mbar_arrive_expect_tx(qd_full(s), 2 * C::TILE + 1024);
                    const uint32_t dst = sQD + s * 2 * C::TILE;
                    for (int x = 0; x < C::NBOX; ++x) {
                        tma_load_4d(dst + x * C::BOX, &tm_q, qd_full(s), x * 64, g.h, qrow, g.b);
                        tma_load_4d(dst + C::TILE + x * C::BOX, &tm_do, qd_full(s), x * 64, g.h, qrow, g.b);
                    }
                    const size_t row = size_t(g.bh) * p.Tp + size_t(qrow);
                    bulk_load(sLSE + s * 1024, p.lse2 + row, 512, qd_full(s));
                    bulk_load(sLSE + s * 1024 + 512, p.delta + row, 512, qd_full(s));
                }
            }
            work_slot_finish(p.work_slot);
            // Drain: make sure no copy is still landing when the CTA exits.
            for (int s = 0; s < C::NSTAGE && s < n; ++s) {
                const int fills = (n - s + C::NSTAGE - 1) / C::NSTAGE;
                mbar_wait(qd_full(s), uint32_t((fills - 1) & 1), abort_flag, p.wait_limit, kStatusTimeoutProducer);
            }
            if (ki > 0) mbar_wait(kv_full, uint32_t((ki - 1) & 1), abort_flag, p.wait_limit, kStatusTimeoutProducer);
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int n = 0, ki = 0;
            for (;; ++ki) {
                const int item = item_consume_thread(ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                                     kStatusTimeoutMma, ok);
                if (!ok || item >= p.n_items) break;
                const BwdItem g = bwd_item(p, item);
                ok = mbar_wait(kv_full, uint32_t(ki & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
                for (int l = 0; l < g.nsteps && ok; ++l, ++n) {
                    const int s = n % C::NSTAGE;
                    const uint32_t par = uint32_t(n & 1);
                    ok = mbar_wait(qd_full(s), (n / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    if (!ok) break;
                    const uint32_t sQ = sQD + s * 2 * C::TILE, sDO = sQ + C::TILE;
                    // S^T overwrites the P^T columns read by dV of the previous step.
                    if (n > 0) {
                        ok = mbar_wait(dv_done, par ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutMma);
                        if (!ok) break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(tS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), C::IDESC_S,
                               kk > 0);
                    }
                    tc_commit(s_full);
                    // dP^T reuses the columns the dQ drain of the previous step reads.
                    if (n > 0) {
                        ok = mbar_wait(dq_free, par ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutMma);
                        if (!ok) break;
                        tc_fence_after();
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(tDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sDO + off, 16, 1024), C::IDESC_S,
                               kk > 0);
                    }
                    tc_commit(dp_full);
                    // dV += P^T dO  (the previous item's epilogue must have read dV / dK first)
                    ok = mbar_wait(p_full, par, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    if (ok && l == 0 && ki > 0)
                        ok = mbar_wait(acc_free, uint32_t((ki - 1) & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)
                        mma_ts(tDV, tS + kk * 8, sdesc_sw128(sDO + kk * 2048, C::BOX, 1024), C::IDESC_ACC,
                               (l > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(dv_done);
                    // dK += dS^T Q ; dQ_i = dS K
                    ok = mbar_wait(ds_full, par, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                        mma_ss(tDK, sdesc_sw128(sDS + off, 16, 1024), sdesc_sw128(sQ + kk * 2048, C::BOX, 1024),
                               C::IDESC_ACC, (l > 0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_ss(tDP, sdesc_sw128(sDS + kk * 2048, C::BOX, 1024),
                               sdesc_sw128(sK + kk * 2048, C::BOX, 1024), C::IDESC_DQ, kk > 0);
                    tc_commit(dq_full);   // also tells the dQ warps that stage s is no longer read by MMAs
                    tc_commit(ds_free);
                }
                if (!ok) break;
                tc_commit(acc_full);   // dV, dK of this item are final
                tc_commit(kv_empty);   // K, V may be replaced by the next item's
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else if (warp < 4) {
        // ------------------------------ key-row warps: P^T and dS^T ------------------------------
        const int row = warp * 32 + lane;
        const uint32_t lane_off = uint32_t(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        bool ok = true;
        int n = 0, ki = 0;
        for (;; ++ki) {
            const int item = item_consume_warp(ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutSoftmax, ok);
            if (!ok || item >= p.n_items) break;
            const BwdItem g = bwd_item(p, item);
            const long long k0 = g.k0;
            const long long kv = k0 + row;
            for (int l = 0; l < g.nsteps && ok; ++l, ++n) {
                const uint32_t par = uint32_t(n & 1);
                const long long q0 = (long long)(g.ilo + l) * C::BM;
                const uint32_t sL = sLSE + (n % C::NSTAGE) * 1024;   // lse*log2e: 128 floats; Delta 512 bytes later
                ok = __all_sync(0xffffffffu,
                                mbar_wait(s_full, par, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                // Both halves of the row (64 columns each) are requested before one wait.
                float pr[C::BM];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tS + lane_off + hh * 64, r0);
                    tmem_ld32(tS + lane_off + hh * 64 + 32, r1);
                    float lz[64];
#pragma unroll
                    for (int gq = 0; gq < 16; ++gq) {
                        const float4 t4 = lds_f32x4(sL + (hh * 64 + gq * 4) * 4);
                        lz[4 * gq] = t4.x;
                        lz[4 * gq + 1] = t4.y;
                        lz[4 * gq + 2] = t4.z;
                        lz[4 * gq + 3] = t4.w;
                    }
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        pr[hh * 64 + i] = ex2_approx(fmaf(__uint_as_float(r0[i]), sl2, -lz[i]));
                        pr[hh * 64 + 32 + i] = ex2_approx(fmaf(__uint_as_float(r1[i]), sl2, -lz[32 + i]));
                    }
                }
                // Tiles that cut the diagonal, the window's far edge or T: keep columns clo..chi of this
                // key row (queries kv .. kv+W-1, below T).  The test is uniform across the CTA.
                const bool full = (k0 + C::BN - 1 <= q0) && (q0 + C::BM - 1 - k0 < W) && (q0 + C::BM <= T);
                if (!full) {
                    const int clo = int(imin_ll(imax_ll(kv - q0, 0), C::BM + 1));
                    const int chi =
                        kv < T ? int(imin_ll(imax_ll(imin_ll(kv + W - 1, (long long)T - 1) - q0, -1), C::BM)) : -1;
#pragma unroll
                    for (int col = 0; col < C::BM; ++col) pr[col] = (col >= clo && col <= chi) ? pr[col] : 0.f;
                }
#pragma unroll
                for (int c = 0; c < C::BM / 64; ++c) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(pr[c * 64 + 2 * i], pr[c * 64 + 2 * i + 1]);
                    tmem_st32(tS + lane_off + c * 32, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full);
                // dS^T = P^T (dP^T - Delta)
                ok = __all_sync(0xffffffffu,
                                mbar_wait(dp_full, par, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                if (n > 0) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(ds_free, par ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                    if (!ok) break;
                }
#pragma unroll
                for (int c = 0; c < C::BM / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tDP + lane_off + c * 32, r);
                    float dz[32];
#pragma unroll
                    for (int gq = 0; gq < 8; ++gq) {
                        const float4 t4 = lds_f32x4(sL + 512 + (c * 32 + gq * 4) * 4);
                        dz[4 * gq] = t4.x;
                        dz[4 * gq + 1] = t4.y;
                        dz[4 * gq + 2] = t4.z;
                        dz[4 * gq + 3] = t4.w;
                    }
                    tmem_ld_wait(r);
                    // 32 query columns = four 16-byte chunks of this key row in the 128B-swizzled tile.
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int col = c * 32 + gq * 8 + 2 * e;
                            const float d0 = pr[col] * (__uint_as_float(r[gq * 8 + 2 * e]) - dz[gq * 8 + 2 * e]);
                            const float d1 =
                                pr[col + 1] * (__uint_as_float(r[gq * 8 + 2 * e + 1]) - dz[gq * 8 + 2 * e + 1]);
                            w[e] = pack_bf16x2(d0, d1);
                        }
                        const int chunk = (c * 32 + gq * 8) >> 3;            // 0..15 across the 128 columns
                        const int box = chunk >> 3, cib = chunk & 7;
                        const uint32_t addr = sDS + box * C::BOX + row * 128 + ((cib ^ (row & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
                                     "r"(w[2]), "r"(w[3])
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (!ok) break;
            // ---- epilogue of the item: dV ----
            ok = __all_sync(0xffffffffu,
                            mbar_wait(acc_full, uint32_t(ki & 1), abort_flag, p.wait_limit, kStatusTimeoutEpilogue));
            if (!ok) break;
            tc_fence_after();
            uint32_t dvr[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tDV + lane_off + c * 32, r);
                tmem_ld_wait(r);
#pragma unroll
                for (int i = 0; i < 32; ++i) dvr[c * 32 + i] = r[i];
            }
            tc_fence_before();
            mbar_arrive(acc_free);
            if (kv < T) {
                __nv_bfloat16* dst = p.dv + ((size_t(g.b) * T + size_t(kv)) * p.H + g.h) * D;
#pragma unroll
                for (int v8 = 0; v8 < D / 8; ++v8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(dvr[v8 * 8 + 0]), __uint_as_float(dvr[v8 * 8 + 1]));
                    w.y = pack_bf16x2(__uint_as_float(dvr[v8 * 8 + 2]), __uint_as_float(dvr[v8 * 8 + 3]));
                    w.z = pack_bf16x2(__uint_as_float(dvr[v8 * 8 + 4]), __uint_as_float(dvr[v8 * 8 + 5]));
                    w.w = pack_bf16x2(__uint_as_float(dvr[v8 * 8 + 6]), __uint_as_float(dvr[v8 * 8 + 7]));
                    *reinterpret_cast<uint4*>(dst + v8 * 8) = w;
                }
            }
        }
    } else {
        // ------------------------------ query-row warps: dQ drain; dK epilogue ------------------------------
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        bool ok = true;
        int n = 0, ki = 0;
        for (;; ++ki) {
            const int item = item_consume_warp(ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutSoftmax, ok);
            if (!ok || item >= p.n_items) break;
            const BwdItem g = bwd_item(p, item);
            for (int l = 0; l < g.nsteps && ok; ++l, ++n) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait(dq_full, uint32_t(n & 1), abort_flag, p.wait_limit, kStatusTimeoutEpilogue));
                if (!ok) break;
                tc_fence_after();
                // Stage the fp32 dQ tile over Q_n / dO_n (no MMA reads them any more): D/32 boxes of
                // 128 rows x 128 bytes, 128-byte swizzled like the TMA box of the reduce.
                const int s = n % C::NSTAGE;
                const uint32_t stg = sQD + s * 2 * C::TILE;
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh) {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tDP + lane_off + hh * 64, r0);
                    tmem_ld32(tDP + lane_off + hh * 64 + 32, r1);
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t* rr = half ? r1 : r0;
                        const int bx = hh * 2 + half;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint32_t addr = stg + bx * C::DQ_BOX + row * 128 + ((j ^ (row & 7)) << 4);
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(rr[j * 4]),
                                         "r"(rr[j * 4 + 1]), "r"(rr[j * 4 + 2]), "r"(rr[j * 4 + 3])
                                         : "memory");
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(dq_free);
                fence_proxy_async_smem();
                mbar_arrive(dq_staged);
                if (threadIdx.x == 128) {
                    ok = mbar_wait(dq_staged, uint32_t(n & 1), abort_flag, p.wait_limit, kStatusTimeoutEpilogue);
                    if (ok) {
                        for (int bx = 0; bx < D / 32; ++bx)
                            tma_reduce_add_4d(&tm_dqacc, stg + bx * C::DQ_BOX, bx * 32, g.h, (g.ilo + l) * C::BM, g.b);
                        bulk_commit_group();
                        bulk_wait_group_read0();   // the stage may be refilled once the reduce has read it
                        mbar_arrive(qd_empty(s));
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
            }
            if (!ok) break;
            // ---- epilogue of the item: scale * dK ----
            ok = __all_sync(0xffffffffu,
                            mbar_wait(acc_full, uint32_t(ki & 1), abort_flag, p.wait_limit, kStatusTimeoutEpilogue));
            if (!ok) break;
            tc_fence_after();
            uint32_t dkr[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tDK + lane_off + c * 32, r);
                tmem_ld_wait(r);
#pragma unroll
                for (int i = 0; i < 32; ++i) dkr[c * 32 + i] = r[i];
            }
            tc_fence_before();
            mbar_arrive(acc_free);
            const long long kv = g.k0 + row;
            if (kv < T) {
                const float sc = p.scale;
                __nv_bfloat16* dst = p.dk + ((size_t(g.b) * T + size_t(kv)) * p.H + g.h) * D;
#pragma unroll
                for (int v8 = 0; v8 < D / 8; ++v8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(dkr[v8 * 8 + 0]) * sc, __uint_as_float(dkr[v8 * 8 + 1]) * sc);
                    w.y = pack_bf16x2(__uint_as_float(dkr[v8 * 8 + 2]) * sc, __uint_as_float(dkr[v8 * 8 + 3]) * sc);
                    w.z = pack_bf16x2(__uint_as_float(dkr[v8 * 8 + 4]) * sc, __uint_as_float(dkr[v8 * 8 + 5]) * sc);
                    w.w = pack_bf16x2(__uint_as_float(dkr[v8 * 8 + 6]) * sc, __uint_as_float(dkr[v8 * 8 + 7]) * sc);
                    *reinterpret_cast<uint4*>(dst + v8 * 8) = w;
                }
            }
        }
        if (threadIdx.x == 128) bulk_wait_group0();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace swa
