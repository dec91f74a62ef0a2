// bwd.cuh -- backward kernels of causal sliding-window attention.
//
// Gradients of sum(dO * O) for the forward in fwd.cuh (training runs through
// flash_attn_func, apidog guide "Train your own ChatGPT", section 5).  With
// P = softmax of the banded scores, Delta_i = sum_d dO_id O_id:
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - Delta),
//   dK = scale * dS^T Q,   dQ = scale * dS K.
//
// Three launches, no atomics and no fp32 gradient accumulator in memory:
//   swa_bwd_pre_kernel    Delta and lse*log2(e) as fp32 rows [B*H, Tp], Tp = 128*ceil(T/128)
//                         (padding: Delta 0, lse +inf), so every 128-query slice is one
//                         aligned 512-byte bulk copy
//   swa_bwd_dkdv_kernel   key-stationary: an item is a 128-row key/value tile of one (b, h);
//                         it walks the query tiles of its band, recomputes P^T from lse and
//                         keeps dV, dK in TMEM (4 MMAs per step)
//   swa_bwd_dq_kernel     query-stationary: an item is a 128-row query tile; it walks the key
//                         tiles of its band, recomputes P and dS and keeps dQ in TMEM
//                         (3 MMAs per step)
// Splitting dQ off costs recomputing S and dP (2 extra MMAs per tile pair) and saves
// the fp32 dQ accumulator round trip: a TMA reduce-add of one 64 KB fp32 dQ partial per
// tile pair is bound by L2 atomics, and it pins the shared memory it reads from.
//
// Both main kernels are persistent (one CTA per SM) and draw head-major items from a
// launch-wide counter (sm100.cuh), so CTAs that run at the same time share a head's
// tiles through L2.  Roles (320 threads):
//   warp 8       TMA producer
//   warp 9       MMA issuer (one thread)
//   warps 0..7   two warpgroups on the same 128 TMEM lanes (one row per lane): warps 0..3
//                take columns 0..63 of the 128-column score tiles, warps 4..7 columns 64..127.
#pragma once

#include "rope.cuh"
#include "sm100.cuh"

namespace swa {

struct BwdParams {
    const float* lse2;    // [B*H, Tp] lse * log2(e), +inf past T
    const float* delta;   // [B*H, Tp], 0 past T
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    int B, T, H;
    int G;                // query heads per K/V head (k, v, dk, dv have H / G heads)
    long long W;
    float scale;
    float scale_log2;
    int n_blk;            // ceil(T / 128)
    int n_items;          // items of this launch: n_blk * B * H (dQ) or n_blk * B * H / G (dK/dV)
    int stream_slot;      // the launch's stream slot: its work counter and status word
    int Tp;               // T rounded up to 128
    long long wait_limit;
    // dQ kernel with kRope: q is the rotated, normalised query; dq is taken back through that
    // prologue at the raw query q_raw (token t at position t) before it is written (rope.cuh)
    const __nv_bfloat16* q_raw;
    const float* rope_cos;  // [max_pos, D/2]
    const float* rope_sin;
    int max_pos;
    float eps;
};

// ---------------------------------------------------------------------------
// Delta_i = sum_d dO_id * O_id and lse * log2(e), as padded fp32 rows.
// One thread per 8 consecutive elements (16 bytes) of a [B,T,H,D] row.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) swa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                          const __nv_bfloat16* __restrict__ dout,
                                                          const float* __restrict__ lse,
                                                          float* __restrict__ lse2, float* __restrict__ delta,
                                                          int B, int T, int H, int Tp) {
    constexpr int LPR = D / 8;   // lanes per row
    const long long nrows = (long long)B * T * H;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
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

// Store 32 fp32 values (bit patterns) of one row as bf16, times `mul`, 16 bytes at a time.
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const uint32_t (&r)[32], float mul) {
    store_row_bf16<32>(dst, reinterpret_cast<const float*>(r), mul);
}

// ===========================================================================
// dK, dV: key-stationary
// ===========================================================================
template <int D>
struct BwdKVCfg {
    static constexpr int BN = 128;                 // key rows per item (MMA M of S^T, dP^T, dV, dK)
    static constexpr int BM = 128;                 // query rows per step
    static constexpr int TILE = 128 * D * 2;
    static constexpr int BOX = 128 * 64 * 2;
    static constexpr int NBOX = D / 64;
    // Q_n ring one deeper than the dO_n ring: S^T(n+1) is issued a step ahead of its use, while
    // the Q and dO slots of step n are freed only once dK(n) has been issued.
    static constexpr int NQ = D == 128 ? 3 : 4;
    static constexpr int NDO = D == 128 ? 2 : 3;   // dO_n with step n's lse*log2e and Delta rows
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = TILE;
    static constexpr int OFF_Q = 2 * TILE;
    static constexpr int OFF_DO = OFF_Q + NQ * TILE;
    static constexpr int OFF_LSE = OFF_DO + NDO * TILE;   // per dO stage: 128 floats lse*log2e, 128 Delta
    static constexpr int OFF_BAR = OFF_LSE + NDO * 2 * 128 * 4;
    // k_full, k_empty, v_full, v_empty, q_full x NQ, q_empty x NQ, do_full x NDO, do_empty x NDO,
    // s_full, s_free, dp_full, p_full, ds_full, mma_done, acc_full, acc_free; item_full, item_empty
    // per ring entry
    static constexpr int NUM_BAR = 4 + 2 * NQ + 2 * NDO + 8 + 2 * kItemRing;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    // Up to 1 KB of slack to align the tile region to 1024 bytes, within the per-block limit;
    // the kernel checks at run time that the aligned layout fits what it was given.
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;     // S^T | dP^T (then packed P^T, dS^T) | dV | dK
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BM, 0, 0);       // K-major A, K-major B
    static constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);      // K-major A, MN-major B
    static_assert(SMEM_USED <= 232448, "shared memory");
};

// Item of the key-stationary kernel: key block kblk of head (b, h); head-major, lowest key
// blocks (the most query tiles under causal masking) first.
// With grouped K/V heads an item is a key tile of one K/V head, and its steps walk the band's
// query tiles for each query head of the group in turn (dK, dV sum over the group).
struct BwdKVItem {
    int b, h;             // batch, K/V head
    long long k0;         // first key row
    int ilo, nband;       // first query tile and number of query tiles in the band
    int nsteps;           // nband * G
};

__device__ __forceinline__ BwdKVItem bwd_kv_item(const BwdParams& p, int item) {
    BwdKVItem it;
    const int kblk = item % p.n_blk;
    const int bhk = item / p.n_blk;
    const int Hk = p.H / p.G;
    it.b = bhk / Hk;
    it.h = bhk % Hk;
    it.k0 = (long long)kblk * 128;
    it.ilo = kblk;
    const int ihi = int(imin_ll(p.T - 1, it.k0 + 127 + p.W - 1) / 128);
    it.nband = ihi - it.ilo + 1;
    it.nsteps = it.nband * p.G;
    return it;
}

// Query head and query tile of step l of a key-stationary item.
__device__ __forceinline__ void bwd_kv_step(const BwdParams& p, const BwdKVItem& g, int l, int& qh, int& qt) {
    qh = g.h * p.G + l / g.nband;
    qt = g.ilo + l % g.nband;
}

// Per step n (one query tile of the item):
//   S^T = K Q^T -> TMEM S,   dP^T = V dO^T -> TMEM dP
//   P^T = exp2(S^T scale log2e - lse2), masked     (row warps, from registers)
//   dS^T = P^T (dP^T - Delta)
//   both packed to bf16 over the dP^T columns each warpgroup has loaded itself: warps 0..3
//   (query columns 0..63) put P^T in TMEM columns 0..31 and dS^T in 32..63 of the dP region,
//   warps 4..7 (query columns 64..127) in 64..95 and 96..127
//   dV += P^T dO,   dK += dS^T Q   (A operands from TMEM)
// The S columns hold S^T only, so S^T(n+1) is issued as soon as the row warps have loaded
// S^T(n), a step ahead of its use; MMA order S(n+1) | dV(n) | dK(n) | dP(n+1).  dP^T(n+1)
// overwrites the packed operands of dV(n) and dK(n): the MMAs one thread issues execute in
// issue order, so it needs no wait for them.  With the left operands of dV and dK in TMEM,
// only Q, dO, K and V are read from shared memory, within the SM's shared-memory bandwidth.
template <int D>
__global__ void __launch_bounds__(BwdKVCfg<D>::THREADS, 1)
swa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
    using C = BwdKVCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) report_status(p.stream_slot, kStatusSmemLayout);
        return;
    }

    const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
    auto sQ = [&](int m) { return base + C::OFF_Q + uint32_t(m % C::NQ) * C::TILE; };     // Q of step m
    auto sDO = [&](int m) { return base + C::OFF_DO + uint32_t(m % C::NDO) * C::TILE; };  // dO of step m
    // lse2 of step m at sLSE(m), Delta 512 bytes later
    auto sLSE = [&](int m) { return base + C::OFF_LSE + uint32_t(m % C::NDO) * 1024u; };
    const uint32_t bar0 = base + C::OFF_BAR;
    const uint32_t k_full = bar0, k_empty = bar0 + 8, v_full = bar0 + 16, v_empty = bar0 + 24;
    auto q_full = [&](int m) { return bar0 + 8u * (4 + m % C::NQ); };
    auto q_empty = [&](int m) { return bar0 + 8u * (4 + C::NQ + m % C::NQ); };
    auto do_full = [&](int m) { return bar0 + 8u * (4 + 2 * C::NQ + m % C::NDO); };
    auto do_empty = [&](int m) { return bar0 + 8u * (4 + 2 * C::NQ + C::NDO + m % C::NDO); };
    const uint32_t bb = bar0 + 8u * (4 + 2 * C::NQ + 2 * C::NDO);
    const uint32_t s_full = bb, s_free = bb + 8, dp_full = bb + 16, p_full = bb + 24, ds_full = bb + 32,
                   mma_done = bb + 40, acc_full = bb + 48, acc_free = bb + 56;
    const uint32_t item_full0 = bb + 64, item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);

    const int T = p.T;
    const long long W = p.W;
    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        for (int s = 0; s < C::NQ; ++s) {
            mbar_init(q_full(s), 1);
            mbar_init(q_empty(s), 1);
        }
        for (int s = 0; s < C::NDO; ++s) {
            mbar_init(do_full(s), 1);
            mbar_init(do_empty(s), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 256);
        mbar_init(dp_full, 1);
        mbar_init(p_full, 256);
        mbar_init(ds_full, 256);
        mbar_init(mma_done, 1);
        mbar_init(acc_full, 1);
        mbar_init(acc_free, 256);
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 1 + 8);   // the MMA thread and warps 0..7
        }
        abort_flag[0] = 0;
        abort_flag[1] = p.stream_slot;   // read by a wait that gives up
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
        // Per item: K, Q_first, V, dO_first, then Q and dO per step, so that S of the item's
        // first step waits for K and one Q tile only.
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            int n = 0, nq = 0, nk = 0, nv = 0;   // steps (dO tiles), Q, K and V tiles issued so far
            bool ok = true;
            for (int ki = 0;; ++ki) {
                const int item =
                    item_produce(p.stream_slot, ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const BwdKVItem g = bwd_kv_item(p, item);
                // K and V are read by this CTA alone: start them towards L2 while the previous
                // item's last steps still hold the shared-memory tiles.
                for (int x = 0; x < C::NBOX; ++x) {
                    tma_prefetch_l2_4d(&tm_k, x * 64, g.h, int(g.k0), g.b);
                    tma_prefetch_l2_4d(&tm_v, x * 64, g.h, int(g.k0), g.b);
                }
                for (int l = 0; l < g.nsteps && ok; ++l) {
                    if (l == 0) {   // K of the previous item is free once its last S completed
                        if (ki > 0 && !(ok = mbar_wait(k_empty, uint32_t((ki - 1) & 1), abort_flag, p.wait_limit,
                                                       kStatusTimeoutProducer)))
                            break;
                        mbar_arrive_expect_tx(k_full, C::TILE);
                        for (int x = 0; x < C::NBOX; ++x)
                            tma_load_4d(sK + x * C::BOX, &tm_k, k_full, x * 64, g.h, int(g.k0), g.b);
                        ++nk;
                    }
                    int qh, qt;
                    bwd_kv_step(p, g, l, qh, qt);
                    const int qrow = qt * C::BM;
                    if (!(ok = mbar_wait(q_empty(n), ((n / C::NQ) & 1) ^ 1u, abort_flag, p.wait_limit,
                                         kStatusTimeoutProducer)))
                        break;
                    mbar_arrive_expect_tx(q_full(n), C::TILE);
                    for (int x = 0; x < C::NBOX; ++x)
                        tma_load_4d(sQ(n) + x * C::BOX, &tm_q, q_full(n), x * 64, qh, qrow, g.b);
                    ++nq;
                    if (l == 0) {   // V of the previous item is free once its last dP completed
                        if (ki > 0 && !(ok = mbar_wait(v_empty, uint32_t((ki - 1) & 1), abort_flag, p.wait_limit,
                                                       kStatusTimeoutProducer)))
                            break;
                        mbar_arrive_expect_tx(v_full, C::TILE);
                        for (int x = 0; x < C::NBOX; ++x)
                            tma_load_4d(sV + x * C::BOX, &tm_v, v_full, x * 64, g.h, int(g.k0), g.b);
                        ++nv;
                    }
                    if (!(ok = mbar_wait(do_empty(n), ((n / C::NDO) & 1) ^ 1u, abort_flag, p.wait_limit,
                                         kStatusTimeoutProducer)))
                        break;
                    mbar_arrive_expect_tx(do_full(n), C::TILE + 1024);
                    for (int x = 0; x < C::NBOX; ++x)
                        tma_load_4d(sDO(n) + x * C::BOX, &tm_do, do_full(n), x * 64, qh, qrow, g.b);
                    const size_t row = (size_t(g.b) * p.H + size_t(qh)) * p.Tp + size_t(qrow);
                    bulk_load(sLSE(n), p.lse2 + row, 512, do_full(n));
                    bulk_load(sLSE(n) + 512, p.delta + row, 512, do_full(n));
                    ++n;
                }
                if (!ok) break;
            }
            work_slot_finish(p.stream_slot);
            // Drain: no copy of this CTA may still be landing when it exits.
            for (int s = 0; s < C::NQ && s < nq; ++s)
                mbar_drain(q_full(s), uint32_t(((nq - s + C::NQ - 1) / C::NQ - 1) & 1), p.wait_limit, p.stream_slot);
            for (int s = 0; s < C::NDO && s < n; ++s)
                mbar_drain(do_full(s), uint32_t(((n - s + C::NDO - 1) / C::NDO - 1) & 1), p.wait_limit, p.stream_slot);
            if (nk > 0) mbar_drain(k_full, uint32_t((nk - 1) & 1), p.wait_limit, p.stream_slot);
            if (nv > 0) mbar_drain(v_full, uint32_t((nv - 1) & 1), p.wait_limit, p.stream_slot);
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int n = 0;
            auto wait = [&](uint32_t bar, int phase) {
                return mbar_wait(bar, uint32_t(phase & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
            };
            // S^T(m) overwrites S^T(m-1), which the row warps have loaded once s_free(m-1) completes.
            auto issue_s = [&](int m, bool last) -> bool {
                if (!wait(q_full(m), m / C::NQ) || (m > 0 && !wait(s_free, m - 1))) return false;
                tc_fence_after();
                const SDesc kd = sdesc_sw128_w(sK, 16, 1024), qd = sdesc_sw128_w(sQ(m), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(tS, kd.lo + off, kd.hi, qd.lo + off, qd.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(s_full);
                if (last) tc_commit(k_empty);
                return true;
            };
            // dP^T(m) overwrites the packed operands of dV(m-1) and dK(m-1), issued earlier by this
            // thread after the row warps had loaded dP^T(m-1).
            auto issue_dp = [&](int m, bool last) -> bool {
                if (!wait(do_full(m), m / C::NDO)) return false;
                tc_fence_after();
                const SDesc vd = sdesc_sw128_w(sV, 16, 1024), od = sdesc_sw128_w(sDO(m), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(tDP, vd.lo + off, vd.hi, od.lo + off, od.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(dp_full);
                if (last) tc_commit(v_empty);
                return true;
            };
            for (int ki = 0;; ++ki) {
                const int item = item_consume_thread(ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                                     kStatusTimeoutMma, ok);
                if (!ok || item >= p.n_items) break;
                const BwdKVItem g = bwd_kv_item(p, item);
                ok = wait(k_full, ki) && issue_s(n, g.nsteps == 1) && wait(v_full, ki) && issue_dp(n, g.nsteps == 1);
                for (int l = 0; l < g.nsteps && ok; ++l, ++n) {
                    const bool more = l + 1 < g.nsteps;
                    if (more && !(ok = issue_s(n + 1, l + 2 == g.nsteps))) break;
                    // dV += P^T dO  (the previous item's epilogue must have read dV / dK)
                    if (!(ok = wait(p_full, n)) || (l == 0 && ki > 0 && !(ok = wait(acc_free, ki - 1)))) break;
                    tc_fence_after();
                    const SDesc od = sdesc_sw128_w(sDO(n), C::BOX, 1024);
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)   // query rows 16kk.. : P^T column pairs of warpgroup kk/4
                        mma_ts_w(tDV, tDP + (kk >> 2) * 64 + (kk & 3) * 8, od.lo + kk * (2048 >> 4), od.hi, C::IDESC_ACC,
                                 (l > 0 || kk > 0) ? 1u : 0u);
                    // dK += dS^T Q
                    if (!(ok = wait(ds_full, n))) break;
                    tc_fence_after();
                    const SDesc qd = sdesc_sw128_w(sQ(n), C::BOX, 1024);
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)
                        mma_ts_w(tDK, tDP + (kk >> 2) * 64 + 32 + (kk & 3) * 8, qd.lo + kk * (2048 >> 4), qd.hi,
                                 C::IDESC_ACC, (l > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(q_empty(n));    // Q_n is read
                    tc_commit(do_empty(n));   // dO_n, lse and Delta of step n are read
                    if (more && !(ok = issue_dp(n + 1, l + 2 == g.nsteps))) break;
                }
                if (!ok) break;
                tc_commit(acc_full);   // dV, dK of this item are final
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else {
        // ------------------------------ key-row warps: P^T, dS^T, epilogue ------------------------------
        // Thread = key row (TMEM lane); warps 0..3 take query columns 0..63, warps 4..7 columns 64..127.
        const int rh = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const float sl2 = p.scale_log2;
        // Epilogue of the pki-th item (index pitem): warps 0..3 write this row's dV,
        // warps 4..7 scale * dK.  It runs at the start of the next item's first step, while
        // that step's S^T and dP^T MMAs (issued earlier) execute.
        auto epilogue = [&](int pki, int pitem) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(acc_full, uint32_t(pki & 1), abort_flag, p.wait_limit,
                                                   kStatusTimeoutEpilogue)))
                return false;
            tc_fence_after();
            const BwdKVItem pg = bwd_kv_item(p, pitem);
            const long long pkv = pg.k0 + row;
            __nv_bfloat16* dst =
                pkv < T ? (rh == 0 ? p.dv : p.dk) + ((size_t(pg.b) * T + size_t(pkv)) * (p.H / p.G) + pg.h) * D
                        : nullptr;
            const uint32_t src = (rh == 0 ? tDV : tDK) + lane_off;
            const float mul = rh == 0 ? 1.f : p.scale;
#pragma unroll
#pragma unroll
            for (int c = 0; c < D / 32; c += 2) {   // 64 columns per wait
                uint32_t a0[32], a1[32];
                tmem_ld32(src + c * 32, a0);
                tmem_ld32(src + c * 32 + 32, a1);
                tmem_ld_wait(a0);
                tmem_ld_wait(a1);
                if (c + 2 == D / 32) {
                    tc_fence_before();
                    mbar_arrive(acc_free);
                }
                if (dst) {
                    store_row32_bf16(dst + c * 32, a0, mul);
                    store_row32_bf16(dst + c * 32 + 32, a1, mul);
                }
            }
            return true;
        };
        bool ok = true;
        int n = 0;
        int prev_ki = -1, prev_item = 0;   // item whose epilogue is still pending
        for (int ki = 0;; ++ki) {
            const int item = item_consume_warp(ki, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutSoftmax, ok);
            if (!ok || item >= p.n_items) break;
            const BwdKVItem g = bwd_kv_item(p, item);
            const long long k0 = g.k0;
            const long long kv = k0 + row;
            for (int l = 0; l < g.nsteps && ok; ++l, ++n) {
                const uint32_t par = uint32_t(n & 1);
                int qh, qt;
                bwd_kv_step(p, g, l, qh, qt);
                const long long q0 = (long long)qt * C::BM;
                const uint32_t sL = sLSE(n) + rh * 256;   // this half's 64 lse2 values
                // The previous item's dV / dK leave TMEM before this item's first dV.
                if (l == 0 && prev_ki >= 0) {
                    if (!(ok = epilogue(prev_ki, prev_item))) break;
                    prev_ki = -1;
                }
                // S^T(n) implies Q_n has landed, not the dO_n stage that carries lse and Delta.
                ok = __all_sync(0xffffffffu,
                                mbar_wait(s_full, par, abort_flag, p.wait_limit, kStatusTimeoutSoftmax) &&
                                    mbar_wait(do_full(n), uint32_t((n / C::NDO) & 1), abort_flag, p.wait_limit,
                                              kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                float pr[64];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tS + lane_off + rh * 64, r0);
                    tmem_ld32(tS + lane_off + rh * 64 + 32, r1);
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
                    tc_fence_before();
                    mbar_arrive(s_free);   // S^T(n+1) may be written
#pragma unroll
                    for (int gq = 0; gq < 8; ++gq) {
                        const float4 a = lds_f32x4(sL + gq * 16);
                        const float4 b = lds_f32x4(sL + 128 + gq * 16);
                        pr[4 * gq + 0] = ex2_approx(fmaf(__uint_as_float(r0[4 * gq + 0]), sl2, -a.x));
                        pr[4 * gq + 1] = ex2_approx(fmaf(__uint_as_float(r0[4 * gq + 1]), sl2, -a.y));
                        pr[4 * gq + 2] = ex2_approx(fmaf(__uint_as_float(r0[4 * gq + 2]), sl2, -a.z));
                        pr[4 * gq + 3] = ex2_approx(fmaf(__uint_as_float(r0[4 * gq + 3]), sl2, -a.w));
                        pr[32 + 4 * gq + 0] = ex2_approx(fmaf(__uint_as_float(r1[4 * gq + 0]), sl2, -b.x));
                        pr[32 + 4 * gq + 1] = ex2_approx(fmaf(__uint_as_float(r1[4 * gq + 1]), sl2, -b.y));
                        pr[32 + 4 * gq + 2] = ex2_approx(fmaf(__uint_as_float(r1[4 * gq + 2]), sl2, -b.z));
                        pr[32 + 4 * gq + 3] = ex2_approx(fmaf(__uint_as_float(r1[4 * gq + 3]), sl2, -b.w));
                    }
                }
                // Tiles that cut the diagonal, the window's far edge or T: keep query columns clo..chi
                // of this key row (queries kv .. kv+W-1, below T).  The test is uniform across the CTA.
                const bool full = (k0 + C::BN - 1 <= q0) && (q0 + C::BM - 1 - k0 < W) && (q0 + C::BM <= T);
                if (!full) {
                    const int clo = int(imin_ll(imax_ll(kv - q0, 0), C::BM + 1)) - rh * 64;
                    const int chi =
                        (kv < T ? int(imin_ll(imax_ll(imin_ll(kv + W - 1, (long long)T - 1) - q0, -1), C::BM)) : -1) -
                        rh * 64;
#pragma unroll
                    for (int col = 0; col < 64; ++col) pr[col] = (col >= clo && col <= chi) ? pr[col] : 0.f;
                }
                ok = __all_sync(0xffffffffu, mbar_wait(dp_full, par, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                // This warpgroup's dP^T columns: the first 32 take packed P^T, the last 32 packed dS^T,
                // each once its dP^T values are in registers.
                const uint32_t tOwn = tDP + lane_off + rh * 64;
                uint32_t w0[16];
                {
                    uint32_t r[32];
                    tmem_ld32(tOwn, r);
                    tmem_ld_wait(r);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pr[hh * 32 + 2 * i], pr[hh * 32 + 2 * i + 1]);
                        tmem_st16(tOwn + hh * 16, pk);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(p_full);
                    // dS^T = P^T (dP^T - Delta), query columns 0..31 of this half
#pragma unroll
                    for (int gq = 0; gq < 8; ++gq) {
                        const float4 a = lds_f32x4(sL + 512 + gq * 16);
                        const int c = 4 * gq;
                        w0[2 * gq] = pack_bf16x2(pr[c] * (__uint_as_float(r[c]) - a.x),
                                                 pr[c + 1] * (__uint_as_float(r[c + 1]) - a.y));
                        w0[2 * gq + 1] = pack_bf16x2(pr[c + 2] * (__uint_as_float(r[c + 2]) - a.z),
                                                     pr[c + 3] * (__uint_as_float(r[c + 3]) - a.w));
                    }
                }
                {
                    uint32_t r[32], w1[16];   // query columns 32..63 of this half
                    tmem_ld32(tOwn + 32, r);
                    tmem_ld_wait(r);
#pragma unroll
                    for (int gq = 0; gq < 8; ++gq) {
                        const float4 a = lds_f32x4(sL + 512 + 128 + gq * 16);
                        const int c = 4 * gq;
                        w1[2 * gq] = pack_bf16x2(pr[32 + c] * (__uint_as_float(r[c]) - a.x),
                                                 pr[33 + c] * (__uint_as_float(r[c + 1]) - a.y));
                        w1[2 * gq + 1] = pack_bf16x2(pr[34 + c] * (__uint_as_float(r[c + 2]) - a.z),
                                                     pr[35 + c] * (__uint_as_float(r[c + 3]) - a.w));
                    }
                    tmem_st16(tOwn + 32, w0);
                    tmem_st16(tOwn + 48, w1);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (!ok) break;
            prev_ki = ki;
            prev_item = item;
        }
        if (ok && prev_ki >= 0) epilogue(prev_ki, prev_item);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ===========================================================================
// dQ: query-stationary
// ===========================================================================
template <int D>
struct BwdQCfg {
    static constexpr int BM = 128;                  // query rows per item (MMA M)
    static constexpr int BN = 128;                  // key rows per step
    static constexpr int TILE = 128 * D * 2;
    static constexpr int BOX = 128 * 64 * 2;
    static constexpr int NBOX = D / 64;
    // Separate K and V rings: K_j is read by S(j) and dQ(j), V_j by dP(j) alone, so with one ring
    // V_{j+1} would wait for the slot dQ(j-1) frees.
    static constexpr int NK = D == 128 ? 3 : 6;
    static constexpr int NV = D == 128 ? 2 : 4;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = TILE;
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + NK * TILE;
    static constexpr int OFF_BAR = OFF_V + NV * TILE;
    // k_full, k_empty per K stage; v_full, v_empty per V stage; q_full, q_empty, do_full, do_empty;
    // s_full x2, s_read x2; dp_full, dp_free, ds_full, dq_full, dq_free, mma_done;
    // item_full, item_empty per ring entry
    static constexpr int NUM_BAR = 2 * (NK + NV) + 4 + 4 + 6 + 2 * kItemRing;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;      // S buffer 0 | S buffer 1 | dP | dQ
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);    // K-major A, K-major B
    static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 0, 1);    // A from TMEM, MN-major B
    static_assert(SMEM_USED <= 232448, "shared memory");
};

// Item of the query-stationary kernel: query tile qt of head (b, h); head-major, latest
// query tiles (the most key tiles under causal masking) first.
struct BwdQItem {
    int b, h, bh, hk;     // batch, query head, b*H + h, K/V head
    long long q0;         // first query row
    int jlo, jhi;         // key tiles of the band
};

__device__ __forceinline__ BwdQItem bwd_q_item(const BwdParams& p, int item) {
    BwdQItem it;
    const int qt = p.n_blk - 1 - item % p.n_blk;
    it.bh = item / p.n_blk;
    it.b = it.bh / p.H;
    it.h = it.bh % p.H;
    it.hk = it.h / p.G;
    it.q0 = (long long)qt * 128;
    it.jlo = int(imax_ll(0, it.q0 - p.W + 1) / 128);
    it.jhi = qt;
    return it;
}

// Per step n (one key tile j of the item):
//   S = Q K_j^T -> TMEM S buffer n%2,   dP = dO V_j^T -> TMEM dP
//   dS = exp2(S scale log2e - lse2) (dP - Delta), masked; bf16 back into the S buffer
//   dQ += dS K_j                (A operand from TMEM)
// The row warps hold dP in registers as soon as they have loaded it, so dP(n+1) is issued
// before dQ(n): MMA order S(n+1) | dP(n+1) | dQ(n).
// kRope: the item's dQ (the gradient at the rotated, normalised query) is taken back through the
// rotary + QK-norm prologue in the epilogue, by warps 0..3 over whole rows: with r = rope(x),
// s = (mean(r^2) + eps)^(-1/2) and dy = dQ:  dr = s dy - (s^3 / D) r (dy . r),  dx = rope^-1(dr).
template <int D, bool kRope = false>
__global__ void __launch_bounds__(BwdQCfg<D>::THREADS, 1)
swa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
    using C = BwdQCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) report_status(p.stream_slot, kStatusSmemLayout);
        return;
    }

    const uint32_t sQ = base + C::OFF_Q, sDO = base + C::OFF_DO;
    auto sK = [&](int m) { return base + C::OFF_K + uint32_t(m % C::NK) * C::TILE; };   // K of step m
    auto sV = [&](int m) { return base + C::OFF_V + uint32_t(m % C::NV) * C::TILE; };   // V of step m
    const uint32_t bar0 = base + C::OFF_BAR;
    auto k_full = [&](int m) { return bar0 + 8u * (m % C::NK); };
    auto k_empty = [&](int m) { return bar0 + 8u * (C::NK + m % C::NK); };
    auto v_full = [&](int m) { return bar0 + 8u * (2 * C::NK + m % C::NV); };
    auto v_empty = [&](int m) { return bar0 + 8u * (2 * C::NK + C::NV + m % C::NV); };
    const uint32_t bb = bar0 + 8u * (2 * (C::NK + C::NV));
    const uint32_t q_full = bb, q_empty = bb + 8, do_full = bb + 16, do_empty = bb + 24;
    auto s_full = [&](int buf) { return bb + 32u + 8u * buf; };
    auto s_read = [&](int buf) { return bb + 48u + 8u * buf; };
    const uint32_t dp_full = bb + 64, dp_free = bb + 72, ds_full = bb + 80, dq_full = bb + 88,
                   dq_free = bb + 96, mma_done = bb + 104;
    const uint32_t item_full0 = bb + 112, item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);

    const int T = p.T;
    const long long W = p.W;
    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(do_full, 1);
        mbar_init(do_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full(b), 1);
            mbar_init(s_read(b), 128);
        }
        mbar_init(dp_full, 1);
        mbar_init(dp_free, 256);
        mbar_init(ds_full, 256);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 256);
        mbar_init(mma_done, 1);
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 1 + 8);   // the MMA thread and warps 0..7
        }
        abort_flag[0] = 0;
        abort_flag[1] = p.stream_slot;   // read by a wait that gives up
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
    auto tSb = [&](int buf) { return tmem + uint32_t(buf) * 128u; };
    const uint32_t tDP = tmem + 256u, tDQ = tmem + 384u;

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        // Order per item: Q, K_jlo, dO, V_jlo, then K_j, V_j per step (Q and dO have their own buffers).
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            int n = 0, nq = 0, ndo = 0, nk = 0, nv = 0;   // steps, Q, dO, K and V tiles issued so far
            bool ok = true;
            auto wait_p = [&](uint32_t bar, int phase) {
                return mbar_wait(bar, uint32_t(phase & 1), abort_flag, p.wait_limit, kStatusTimeoutProducer);
            };
            for (int qi = 0;; ++qi) {
                const int item =
                    item_produce(p.stream_slot, qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const BwdQItem g = bwd_q_item(p, item);
                // Q and dO are read by this CTA alone: start them towards L2 while the previous
                // item's last steps still hold the shared-memory tiles.
                for (int x = 0; x < C::NBOX; ++x) {
                    tma_prefetch_l2_4d(&tm_q, x * 64, g.h, int(g.q0), g.b);
                    tma_prefetch_l2_4d(&tm_do, x * 64, g.h, int(g.q0), g.b);
                }
                for (int j = g.jlo; j <= g.jhi; ++j, ++n) {
                    if (j == g.jlo) {
                        if (qi > 0 && !(ok = wait_p(q_empty, qi - 1))) break;
                        mbar_arrive_expect_tx(q_full, C::TILE);
                        for (int x = 0; x < C::NBOX; ++x) tma_load_4d(sQ + x * C::BOX, &tm_q, q_full, x * 64, g.h, int(g.q0), g.b);
                        ++nq;
                    }
                    if (!(ok = wait_p(k_empty(n), n / C::NK + 1))) break;   // first pass: the phase before 0
                    mbar_arrive_expect_tx(k_full(n), C::TILE);
                    for (int x = 0; x < C::NBOX; ++x) tma_load_4d(sK(n) + x * C::BOX, &tm_k, k_full(n), x * 64, g.hk, j * C::BN, g.b);
                    ++nk;
                    if (j == g.jlo) {
                        if (qi > 0 && !(ok = wait_p(do_empty, qi - 1))) break;
                        mbar_arrive_expect_tx(do_full, C::TILE);
                        for (int x = 0; x < C::NBOX; ++x) tma_load_4d(sDO + x * C::BOX, &tm_do, do_full, x * 64, g.h, int(g.q0), g.b);
                        ++ndo;
                    }
                    if (!(ok = wait_p(v_empty(n), n / C::NV + 1))) break;
                    mbar_arrive_expect_tx(v_full(n), C::TILE);
                    for (int x = 0; x < C::NBOX; ++x) tma_load_4d(sV(n) + x * C::BOX, &tm_v, v_full(n), x * 64, g.hk, j * C::BN, g.b);
                    ++nv;
                }
                if (!ok) break;
            }
            work_slot_finish(p.stream_slot);
            // Drain: no copy of this CTA may still be landing when it exits.
            for (int s = 0; s < C::NK && s < nk; ++s) mbar_drain(k_full(s), uint32_t(((nk - s + C::NK - 1) / C::NK - 1) & 1), p.wait_limit, p.stream_slot);
            for (int s = 0; s < C::NV && s < nv; ++s) mbar_drain(v_full(s), uint32_t(((nv - s + C::NV - 1) / C::NV - 1) & 1), p.wait_limit, p.stream_slot);
            if (nq > 0) mbar_drain(q_full, uint32_t((nq - 1) & 1), p.wait_limit, p.stream_slot);
            if (ndo > 0) mbar_drain(do_full, uint32_t((ndo - 1) & 1), p.wait_limit, p.stream_slot);
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int n = 0;   // steps (all items)
            auto wait = [&](uint32_t bar, int phase) {
                return mbar_wait(bar, uint32_t(phase & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
            };
            // S(m) goes to buffer m%2, which held dS(m-2) for dQ(m-2): issued earlier by this thread.
            auto issue_s = [&](int m, bool last) -> bool {
                if (!wait(k_full(m), m / C::NK)) return false;
                tc_fence_after();
                const SDesc qd = sdesc_sw128_w(sQ, 16, 1024), kd = sdesc_sw128_w(sK(m), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(tSb(m & 1), qd.lo + off, qd.hi, kd.lo + off, kd.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(s_full(m & 1));
                if (last) tc_commit(q_empty);
                return true;
            };
            // dP(m) overwrites dP(m-1), which the row warps have loaded once dp_free(m-1) completes.
            auto issue_dp = [&](int m, bool last) -> bool {
                if (!wait(v_full(m), m / C::NV) || (m > 0 && !wait(dp_free, m - 1))) return false;
                tc_fence_after();
                const SDesc od = sdesc_sw128_w(sDO, 16, 1024), vd = sdesc_sw128_w(sV(m), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(tDP, od.lo + off, od.hi, vd.lo + off, vd.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(dp_full);
                tc_commit(v_empty(m));   // V_j is read by this dP only
                if (last) tc_commit(do_empty);
                return true;
            };
            for (int qi = 0;; ++qi) {
                const int item = item_consume_thread(qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                                     kStatusTimeoutMma, ok);
                if (!ok || item >= p.n_items) break;
                const BwdQItem g = bwd_q_item(p, item);
                const int nsteps = g.jhi - g.jlo + 1;
                ok = wait(q_full, qi) && issue_s(n, nsteps == 1) && wait(do_full, qi) && issue_dp(n, nsteps == 1);
                for (int l = 0; l < nsteps && ok; ++l, ++n) {
                    const bool more = l + 1 < nsteps;
                    if (more && !(ok = issue_s(n + 1, l + 2 == nsteps) && issue_dp(n + 1, l + 2 == nsteps))) break;
                    // dQ += dS K_j  (the previous item's epilogue must have read dQ)
                    if (!(ok = wait(ds_full, n)) || (l == 0 && qi > 0 && !(ok = wait(dq_free, qi - 1)))) break;
                    tc_fence_after();
                    const SDesc kd = sdesc_sw128_w(sK(n), C::BOX, 1024);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_ts_w(tDQ, tSb(n & 1) + kk * 8, kd.lo + kk * (2048 >> 4), kd.hi, C::IDESC_DQ,
                                 (l > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(k_empty(n));   // K_j: read by S(n) and dQ(n)
                }
                if (!ok) break;
                tc_commit(dq_full);   // dQ of this item is final
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else {
        // ------------------------------ query-row warps: dS, epilogue ------------------------------
        // Thread = query row (TMEM lane); warps 0..3 take key columns 0..63, warps 4..7 columns 64..127.
        const int rh = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const float sl2 = p.scale_log2;
        // Epilogue of item pqi (this row's half of dQ at dst, null past T): dQ = scale * acc.  It
        // runs after P of the next item's first step, so that P overlaps the last dQ MMA.
        auto epilogue = [&](int pqi, __nv_bfloat16* dst) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(dq_full, uint32_t(pqi & 1), abort_flag, p.wait_limit,
                                                   kStatusTimeoutEpilogue)))
                return false;
            tc_fence_after();
            uint32_t acc[D / 64][32];
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_ld32(tDQ + lane_off + rh * (D / 2) + c * 32, acc[c]);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_ld_wait(acc[c]);
            tc_fence_before();
            mbar_arrive(dq_free);
            if (dst) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c) store_row32_bf16(dst + c * 32, acc[c], p.scale);
            }
            return true;
        };
        // kRope epilogue of item pqi, query row pq of head (pb, ph): warps 4..7 only release the
        // accumulator; warps 0..3 read whole rows (pairs (i, i + D/2) together) in two passes, the
        // first for the row's two sums, the second for the output.
        auto epilogue_rope = [&](int pqi, long long pq, int pb, int ph) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(dq_full, uint32_t(pqi & 1), abort_flag, p.wait_limit,
                                                   kStatusTimeoutEpilogue)))
                return false;
            tc_fence_after();
            if (rh == 0) {
                const uint32_t src = tDQ + lane_off;
                const bool in = pq < T, posok = pq < p.max_pos;
                const size_t roff = ((size_t(pb) * T + size_t(in ? pq : 0)) * p.H + ph) * D;
                const __nv_bfloat16* xr = p.q_raw + roff;
                __nv_bfloat16* dst = p.dq + roff;
                const float* cr = p.rope_cos + size_t(posok ? pq : 0) * (D / 2);
                const float* sr = p.rope_sin + size_t(posok ? pq : 0) * (D / 2);
                if (in && !posok) report_status(p.stream_slot, kStatusPositionRange);
                float sxx = 0.f, sdr = 0.f, s_ = 0.f, k3 = 0.f;
#pragma unroll 1
                for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
                    for (int c = 0; c < D / 2; c += 32) {
                        uint32_t a1[32], a2[32];   // dQ columns c.. and their partners c + D/2..
                        __syncwarp();              // the TMEM loads are warp-collective
                        tmem_ld32(src + c, a1);
                        tmem_ld32(src + D / 2 + c, a2);
                        tmem_ld_wait(a1);
                        tmem_ld_wait(a2);
                        if (!in) continue;
                        if (!posok) {   // no table row: the gradient at the rotated query, as is
                            if (pass == 1) {
                                store_row32_bf16(dst + c, a1, p.scale);
                                store_row32_bf16(dst + D / 2 + c, a2, p.scale);
                            }
                            continue;
                        }
#pragma unroll
                        for (int v = 0; v < 32; v += 8) {
                            float x1[8], x2[8];
                            bf16x8_unpack(*reinterpret_cast<const uint4*>(xr + c + v), x1);
                            bf16x8_unpack(*reinterpret_cast<const uint4*>(xr + D / 2 + c + v), x2);
                            const float4 c0 = *reinterpret_cast<const float4*>(cr + c + v);
                            const float4 c1 = *reinterpret_cast<const float4*>(cr + c + v + 4);
                            const float4 s0 = *reinterpret_cast<const float4*>(sr + c + v);
                            const float4 s1 = *reinterpret_cast<const float4*>(sr + c + v + 4);
                            const float co[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                            const float si[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            float o1[8], o2[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float r1 = fmaf(x1[i], co[i], -x2[i] * si[i]);
                                const float r2 = fmaf(x1[i], si[i], x2[i] * co[i]);
                                const float dy1 = __uint_as_float(a1[v + i]) * p.scale;
                                const float dy2 = __uint_as_float(a2[v + i]) * p.scale;
                                if (pass == 0) {
                                    sxx = fmaf(r1, r1, fmaf(r2, r2, sxx));
                                    sdr = fmaf(dy1, r1, fmaf(dy2, r2, sdr));
                                } else {
                                    const float dr1 = fmaf(s_, dy1, -k3 * r1), dr2 = fmaf(s_, dy2, -k3 * r2);
                                    o1[i] = fmaf(dr1, co[i], dr2 * si[i]);    // rotated back
                                    o2[i] = fmaf(dr2, co[i], -dr1 * si[i]);
                                }
                            }
                            if (pass == 1) {
                                *reinterpret_cast<uint4*>(dst + c + v) = bf16x8_pack(o1);
                                *reinterpret_cast<uint4*>(dst + D / 2 + c + v) = bf16x8_pack(o2);
                            }
                        }
                    }
                    if (pass == 0) {
                        const float ms = sxx * (1.f / D) + p.eps;
                        s_ = ms > 0.f ? rsqrtf(ms) : 0.f;
                        k3 = s_ * s_ * s_ * (1.f / D) * sdr;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(dq_free);
            return true;
        };
        bool ok = true;
        int n = 0;
        int prev_qi = -1;                  // item whose epilogue is still pending
        __nv_bfloat16* prev_dst = nullptr;
        long long prev_q = 0;              // kRope: its query row and head
        int prev_b = 0, prev_h = 0;
        for (int qi = 0;; ++qi) {
            const int item = item_consume_warp(qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutSoftmax, ok);
            if (!ok || item >= p.n_items) break;
            const BwdQItem g = bwd_q_item(p, item);
            const long long q = g.q0 + row;
            const size_t prow = size_t(g.bh) * p.Tp + size_t(q);   // padded rows: in bounds for every q
            const float lse2_q = p.lse2[prow];
            const float delta_q = p.delta[prow];
            for (int j = g.jlo; j <= g.jhi && ok; ++j, ++n) {
                const int buf = n & 1;
                const uint32_t ph = uint32_t((n >> 1) & 1);
                if (kRope && j == g.jlo && prev_qi >= 0) {   // before this step's scores: registers are free
                    if (!(ok = epilogue_rope(prev_qi, prev_q, prev_b, prev_h))) break;
                    prev_qi = -1;
                }
                ok = __all_sync(0xffffffffu,
                                mbar_wait(s_full(buf), ph, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                float pr[64];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tSb(buf) + lane_off + rh * 64, r0);
                    tmem_ld32(tSb(buf) + lane_off + rh * 64 + 32, r1);
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        pr[i] = ex2_approx(fmaf(__uint_as_float(r0[i]), sl2, -lse2_q));
                        pr[32 + i] = ex2_approx(fmaf(__uint_as_float(r1[i]), sl2, -lse2_q));
                    }
                }
                // Packed dS of key columns 64..127 goes to TMEM columns 32..63 of the buffer, which hold
                // S of key columns 32..63 that warps 0..3 read: those warps say when they have.
                if (rh == 0) {
                    tc_fence_before();
                    mbar_arrive(s_read(buf));
                }
                // Tiles that cut the diagonal or the window's far edge: keep key columns clo..chi of this
                // query row (keys q-W+1 .. q).  The test is uniform across the CTA.
                const long long k0 = (long long)j * C::BN;
                const bool full = (k0 + C::BN - 1 <= g.q0) && (k0 > g.q0 + C::BM - 1 - W);
                if (!full) {
                    const int chi = int(imin_ll(imax_ll(q - k0, -1), C::BN)) - rh * 64;
                    const int clo = int(imin_ll(imax_ll(q - W + 1 - k0, 0), C::BN + 1)) - rh * 64;
#pragma unroll
                    for (int c = 0; c < 64; ++c) pr[c] = (c >= clo && c <= chi) ? pr[c] : 0.f;
                }
                if (!kRope && j == g.jlo && prev_qi >= 0) {
                    if (!(ok = epilogue(prev_qi, prev_dst))) break;
                    prev_qi = -1;
                }
                ok = __all_sync(0xffffffffu,
                                mbar_wait(dp_full, uint32_t(n & 1), abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                uint32_t pk[32];
                {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tDP + lane_off + rh * 64, r0);
                    tmem_ld32(tDP + lane_off + rh * 64 + 32, r1);
                    tmem_ld_wait(r0);
                    tmem_ld_wait(r1);
                    tc_fence_before();
                    mbar_arrive(dp_free);   // dP(n+1) may be written
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        pk[i] = pack_bf16x2(pr[2 * i] * (__uint_as_float(r0[2 * i]) - delta_q),
                                            pr[2 * i + 1] * (__uint_as_float(r0[2 * i + 1]) - delta_q));
                        pk[16 + i] = pack_bf16x2(pr[32 + 2 * i] * (__uint_as_float(r1[2 * i]) - delta_q),
                                                 pr[33 + 2 * i] * (__uint_as_float(r1[2 * i + 1]) - delta_q));
                    }
                }
                if (rh == 1) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(s_read(buf), ph, abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                    if (!ok) break;
                    tc_fence_after();
                }
                tmem_st32(tSb(buf) + lane_off + rh * 32, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(ds_full);
            }
            if (!ok) break;
            prev_qi = qi;
            prev_dst = q < T ? p.dq + ((size_t(g.b) * T + size_t(q)) * p.H + g.h) * D + rh * (D / 2) : nullptr;
            prev_q = q;
            prev_b = g.b;
            prev_h = g.h;
        }
        if (ok && prev_qi >= 0) {
            if (kRope)
                epilogue_rope(prev_qi, prev_q, prev_b, prev_h);
            else
                epilogue(prev_qi, prev_dst);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace swa
