// fwd.cuh -- forward kernels: O and logsumexp of causal sliding-window attention.
//
// The operation is the one nanochat's GPT calls once per layer,
// flash_attn_func(q, k, v, causal=True, window_size=W) (apidog guide "Train
// your own ChatGPT", section 5 "Flash Attention unification"), with the
// per-layer short/long windows of the "SSSL" pattern (same guide, section 1
// "GPT model", architecture features).  Query i attends to keys
// j in (i - W, i]; W >= T is full causal.
//
// Persistent: one CTA per SM draws work items (query block of 256 rows, b, h) from a
// launch-wide counter; items are head-major so that concurrent CTAs share a head's K/V
// in L2, heaviest query blocks of a head first.  An item is two 128-row query tiles; the CTA
// walks the key/value tiles that intersect the band of either tile:
//   warp 8      TMA producer: Q tiles of each item, then K_j, V_j into a ring
//               of stages that runs on across items
//   warp 9      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM, then
//               O_t += P_t V_j with P_t read from TMEM
//   warps 0..7  two softmax warpgroups, one per query tile; thread = row.
//               Online softmax in the exp2 domain, P written back to TMEM as
//               bf16 over the first half of S_t's columns, O rescaled in TMEM
//               only when a warp's running max grows by more than 2^8.
// The next item's Q load and first S MMAs overlap the current item's last PV
// MMAs and epilogue.  Key tiles entirely outside the band are never loaded;
// only tiles that cut the diagonal or the window's left edge are masked.
// That is swa_fwd_kernel, the one MMA issuer moving both tiles in lockstep.
// swa_fwd_short_kernel (further down) serves windows shorter than the sequence:
// one issuer per tile and a downward walk, so consecutive items overlap.  Both
// use the same softmax warpgroup (fwd_softmax_warpgroup).
#pragma once

#include "rope.cuh"
#include "sm100.cuh"

namespace swa {

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                  // query rows per tile (one MMA M)
    static constexpr int BN = 128;                  // key rows per tile
    static constexpr int NQ = 2;                    // query tiles per item
    static constexpr int TILE = 128 * D * 2;        // bytes of a 128 x D bf16 tile
    static constexpr int BOX = 128 * 64 * 2;        // one TMA box: 128 rows x 64 columns
    static constexpr int NBOX = D / 64;
    static constexpr int NQBUF = 1;                 // Q buffers (2: the next item's Q loads a whole item ahead)
    static constexpr int NSTAGE = D == 128 ? 5 : 8; // K/V ring (a stage holds one K or one V tile)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = NQBUF * NQ * TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    // kv_full, kv_empty per stage; q_full, q_empty per Q buffer; s_full, p_full, o_full, o_free per
    // tile; q_ready per Q buffer; mma_done; item_full, item_empty per entry of the item ring
    static constexpr int NUM_BAR = 2 * NSTAGE + 3 * NQBUF + 4 * NQ + 1 + 2 * kItemRing;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    // Up to 1 KB of slack to align the tile region to 1024 bytes, within the per-block limit;
    // the kernel checks at run time that the aligned layout fits what it was given.
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 320;
    // With the rotary + QK-norm prologue two more warps rotate and normalise each Q tile in shared
    // memory (12 warps: still three per SM sub-partition, so the same register budget).
    static constexpr int threads(bool rope) { return rope ? THREADS + 64 : THREADS; }
    static constexpr uint32_t TMEM_COLS = 512;      // S0 | S1 | O0 | O1
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(SMEM_USED <= 232448, "shared memory");
};

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    int B, T, H;          // T: query rows per sequence
    int G;                // query heads per K/V head (K, V have H / G heads)
    // Chunked prefill (kernel instantiated with kOffset): query row t of sequence b sits at
    // absolute position q_offset[b] + t, and keys are absolute positions in K / V (a KV cache).
    const int* q_offset;
    long long W;
    float scale_log2;     // softmax scale * log2(e)
    int n_qblk;           // ceil(T / 256)
    int n_items;          // n_qblk * B * H
    int stream_slot;      // the launch's stream slot: its work counter and status word
    long long wait_limit; // clock cycles before a wait gives up
    // kRope: Q rows are rotated and normalised at their positions (q_offset[b] + t) before any S MMA
    // reads them (rope.cuh); store_qrot: the rotated tiles are also written through tm_qr
    const float* rope_cos;   // [max_pos, D/2]
    const float* rope_sin;
    int max_pos;
    float eps;
    int store_qrot;
};

// Geometry of one work item: query block qblk of head (b, h).
struct FwdItem {
    int b, h, hk;         // batch, query head, K/V head
    int L;                // absolute position of query row 0 of this sequence
    long long q0;         // first query row of tile 0 (tile 1 starts 128 rows later)
    bool valid1;          // tile 1 has rows below T
    int jlo0, jhi0, jlo1, jhi1, jbeg, jend;
};

// Items are head-major (all query blocks of one (b, h), then the next head), so the CTAs that
// run at the same time read the same head's K/V tiles and share them through L2; within a
// head the heaviest (latest) query blocks come first.
template <bool kOffset>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int item) {
    FwdItem it;
    const int bh = item / p.n_qblk;
    const int qblk = p.n_qblk - 1 - item % p.n_qblk;
    it.b = bh / p.H;
    it.h = bh % p.H;
    it.hk = it.h / p.G;
    it.L = kOffset ? max(0, p.q_offset[it.b]) : 0;
    it.q0 = (long long)qblk * 256;
    it.valid1 = it.q0 + 128 < p.T;
    // key tiles by absolute position: query row t sees keys (L+t-W, L+t]
    it.jlo0 = int(imax_ll(0, it.L + it.q0 - p.W + 1) / 128);
    it.jhi0 = int((it.L + imin_ll(it.q0 + 127, p.T - 1)) / 128);
    it.jlo1 = int(imax_ll(0, it.L + it.q0 + 128 - p.W + 1) / 128);
    it.jhi1 = int((it.L + imin_ll(it.q0 + 255, p.T - 1)) / 128);
    it.jbeg = it.jlo0;
    it.jend = it.valid1 ? it.jhi1 : it.jhi0;
    return it;
}

// Softmax warpgroup of query tile t = warp / 4 (warps 0..7 of a forward kernel), for every item
// of the CTA: thread = row; online softmax of S_t in the exp2 domain, P_t written back to TMEM as
// bf16 over the first half of S_t's columns, O_t rescaled in TMEM only when a warp's running max
// grows by more than 2^8, then the epilogue O / l and lse.  kDown: the item's key tiles arrive
// from the band's last to its first (the order the kernel's MMAs use).  The barriers are those of
// tile t.
template <int D, bool kOffset, bool kDown>
__device__ __forceinline__ void fwd_softmax_warpgroup(const FwdParams& p, uint32_t tS_t, uint32_t tO_t,
                                                      uint32_t s_full, uint32_t p_full, uint32_t o_full,
                                                      uint32_t o_free, volatile int* ring, uint32_t item_full0,
                                                      uint32_t item_empty0, volatile int* abort_flag) {
using C = FwdCfg<D>;
const int T = p.T;
const long long W = p.W;
const int warp = warp_id(), lane = lane_id();
const int t = warp >> 2;            // query tile of this warpgroup
const int quarter = warp & 3;       // TMEM lane quarter this warp may access
const int row = quarter * 32 + lane;
const uint32_t lane_off = uint32_t(quarter * 32) << 16;
const uint32_t tS = tS_t + lane_off, tO = tO_t + lane_off;
    const float sl2 = p.scale_log2;
    int ns = 0;      // S tiles consumed so far (all items): parity of s_full / o_full
    bool ok = true;
    for (int k = 0;; ++k) {
        const int item = item_consume_warp(k, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                           kStatusTimeoutSoftmax, ok);
        if (!ok || item >= p.n_items) break;
        const FwdItem g = fwd_item<kOffset>(p, item);
        if (t == 1 && !g.valid1) continue;
        const long long qt0 = g.q0 + t * 128;    // first row of this tile
        const long long q = qt0 + row;           // query row of this thread (position g.L + q)
        const int jlo = t ? g.jlo1 : g.jlo0, jhi = t ? g.jhi1 : g.jhi0;
        float m_run = -INFINITY, l_run = 0.f;
        int nloc = 0;
        for (int j = kDown ? jhi : jlo; (kDown ? j >= jlo : j <= jhi) && ok; j += kDown ? -1 : 1, ++ns, ++nloc) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(s_full, uint32_t(ns & 1), abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
            if (!ok) break;
            tc_fence_after();
            // All 128 columns are requested before the single wait, so the TMEM load
            // latency is paid once per tile.
            float s[C::BN];
            {
                uint32_t r0[32], r1[32], r2[32], r3[32];
                tmem_ld32(tS, r0);
                tmem_ld32(tS + 32, r1);
                tmem_ld32(tS + 64, r2);
                tmem_ld32(tS + 96, r3);
                tmem_ld_wait(r0);
                tmem_ld_wait(r1);
                tmem_ld_wait(r2);
                tmem_ld_wait(r3);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    s[i] = __uint_as_float(r0[i]);
                    s[32 + i] = __uint_as_float(r1[i]);
                    s[64 + i] = __uint_as_float(r2[i]);
                    s[96 + i] = __uint_as_float(r3[i]);
                }
            }
            // Tiles that cut the diagonal or the window's left edge: keep columns clo..chi of this
            // row (keys k0+c with q-W < k0+c <= q).  The test is uniform across the CTA.
            // k0: the key tile's first position, counted like the query rows (absolute - g.L)
            const long long k0 = (long long)j * C::BN - g.L;
            const bool full = (k0 + C::BN - 1 <= qt0) && (k0 > qt0 + C::BM - 1 - W);
            if (!full) {
                const int chi = int(imin_ll(imax_ll(q - k0, -1), C::BN));
                const int clo = int(imin_ll(imax_ll(q - W + 1 - k0, 0), C::BN + 1));
#pragma unroll
                for (int c = 0; c < C::BN; ++c) s[c] = (c >= clo && c <= chi) ? s[c] : -INFINITY;
            }
            // Row max and row sum over 8 independent partials (short dependency chains).
            float mp[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
            for (int c = 8; c < C::BN; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
            const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                   fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
            const float m_tile = mx * sl2;
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + 8.0f;
            const bool warp_need = __any_sync(0xffffffffu, need);
            const float m_use = warp_need ? m_new : m_run;
            const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
            const float alpha = (m_use == -INFINITY) ? 1.f : ex2_approx(m_run - m_use);
            float sp[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) sp[u] = 0.f;
#pragma unroll
            for (int c = 0; c < C::BN / 64; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p0 = ex2_approx(fmaf(s[c * 64 + 2 * i], sl2, -m_sub));
                    const float p1 = ex2_approx(fmaf(s[c * 64 + 2 * i + 1], sl2, -m_sub));
                    sp[(2 * i) & 7] += p0;
                    sp[(2 * i + 1) & 7] += p1;
                    // bf16 rounding of P: one cvt per pair in the short-window kernel, three integer
                    // instructions (round half up) in the lockstep one; each measured the faster there.
                    pk[i] = kDown ? pack_bf16x2(p0, p1) : pack_bf16x2_alu(p0, p1);
                }
                tmem_st32(tS + c * 32, pk);
            }
            const float rowsum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
            l_run = l_run * alpha + rowsum;
            tmem_st_wait();
            if (warp_need && nloc > 0) {
                // O_t holds the sum over the key tiles walked before j: wait for their PV_t, then rescale.
                ok = __all_sync(0xffffffffu, mbar_wait(o_full, uint32_t((ns - 1) & 1), abort_flag,
                                                       p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tO + c * 32, r);
                    tmem_ld_wait(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tO + c * 32, r);
                }
                tmem_st_wait();
            }
            m_run = m_use;
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (!ok || nloc == 0) break;
        // ---- epilogue: O = O / l, lse = ln(sum exp S) ----
        ok = __all_sync(0xffffffffu, mbar_wait(o_full, uint32_t((ns - 1) & 1), abort_flag, p.wait_limit,
                                               kStatusTimeoutEpilogue));
        if (!ok) break;
        tc_fence_after();
        float ov[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[c * 32 + i] = __uint_as_float(r[i]);
        }
        tc_fence_before();
        mbar_arrive(o_free);   // the next item's first PV may overwrite O_t now
        const long long qrow = q;
        if (qrow < T) {
            const float inv_l = 1.f / l_run;
            __nv_bfloat16* orow = p.o + ((size_t(g.b) * T + size_t(qrow)) * p.H + g.h) * D;
            store_row_bf16<D>(orow, ov, inv_l);
            p.lse[(size_t(g.b) * p.H + g.h) * T + qrow] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
        }
    }
}

// kOffset: chunked prefill (query rows start at q_offset[b]); false for training, where the
// offset is zero and costs nothing.  kRope: the rotary + QK-norm prologue of the queries runs
// inside the kernel (warps 10 and 11), on each Q tile in shared memory between its load and the
// first S MMA; tm_qr then describes where the rotated queries are stored (when p.store_qrot).
template <int D, bool kOffset = false, bool kRope = false>
__global__ void __launch_bounds__(FwdCfg<D>::threads(kRope), 1)
swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qr,
               const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) report_status(p.stream_slot, kStatusSmemLayout);
        return;
    }

    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (C::NSTAGE + s); };
    auto q_full = [&](int qb) { return bar0 + 8u * (2 * C::NSTAGE + qb); };
    auto q_empty = [&](int qb) { return bar0 + 8u * (2 * C::NSTAGE + C::NQBUF + qb); };
    const uint32_t bt = bar0 + 8u * (2 * C::NSTAGE + 2 * C::NQBUF);   // per-tile barriers start here
    auto s_full = [&](int t) { return bt + 8u * t; };
    auto p_full = [&](int t) { return bt + 8u * (C::NQ + t); };
    auto o_full = [&](int t) { return bt + 8u * (2 * C::NQ + t); };
    auto o_free = [&](int t) { return bt + 8u * (3 * C::NQ + t); };
    auto q_ready = [&](int qb) { return bt + 8u * (4 * C::NQ + qb); };   // kRope: Q rotated in place
    const uint32_t mma_done = bt + 8u * (4 * C::NQ + C::NQBUF);
    const uint32_t item_full0 = mma_done + 8u, item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);

    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int qb = 0; qb < C::NQBUF; ++qb) {
            mbar_init(q_full(qb), 1);
            mbar_init(q_empty(qb), kRope ? 2 : 1);   // the S MMAs have read it (and the q_rot store)
            mbar_init(q_ready(qb), 64);
        }
        for (int t = 0; t < C::NQ; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_full(t), 1);
            mbar_init(o_free(t), 128);
        }
        mbar_init(mma_done, 1);
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 1 + 8 + (kRope ? 2 : 0));   // MMA thread, softmax (+ prologue) warps
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
    const uint32_t tS0 = tmem, tS1 = tmem + 128u;
    const uint32_t tO0 = tmem + 256u, tO1 = tmem + 256u + uint32_t(D);

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int it = 0, qi = 0;
            bool ok = true;
            for (;; ++qi) {
                const int item =
                    item_produce(p.stream_slot, qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<kOffset>(p, item);
                // A Q buffer is free once the S MMAs of the item that used it completed.
                const int qb = qi % C::NQBUF;
                if (qi >= C::NQBUF) {
                    ok = mbar_wait(q_empty(qb), uint32_t(((qi / C::NQBUF) - 1) & 1), abort_flag, p.wait_limit,
                                   kStatusTimeoutProducer);
                    if (!ok) break;
                }
                mbar_arrive_expect_tx(q_full(qb), (g.valid1 ? 2 : 1) * C::TILE);
                for (int t = 0; t < (g.valid1 ? 2 : 1); ++t)
                    for (int x = 0; x < C::NBOX; ++x)
                        tma_load_4d(sQ + (qb * C::NQ + t) * C::TILE + x * C::BOX, &tm_q, q_full(qb), x * 64, g.h,
                                    int(g.q0) + t * 128, g.b);
                for (int j = g.jbeg; j <= g.jend && ok; ++j) {
                    for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
                        const int s = it % C::NSTAGE;
                        const uint32_t ph = (it / C::NSTAGE) & 1;
                        ok = mbar_wait(kv_empty(s), ph ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutProducer);
                        if (!ok) break;
                        mbar_arrive_expect_tx(kv_full(s), C::TILE);
                        const CUtensorMap* m = kv ? &tm_v : &tm_k;
                        for (int x = 0; x < C::NBOX; ++x)
                            tma_load_4d(sKV + s * C::TILE + x * C::BOX, m, kv_full(s), x * 64, g.hk, j * C::BN, g.b);
                    }
                }
            }
            work_slot_finish(p.stream_slot);
            // Drain: make sure no copy is still landing when the CTA exits.
            for (int s = 0; s < C::NSTAGE && s < it; ++s) {
                const int fills = (it - s + C::NSTAGE - 1) / C::NSTAGE;
                mbar_drain(kv_full(s), uint32_t((fills - 1) & 1), p.wait_limit, p.stream_slot);
            }
            for (int qb = 0; qb < C::NQBUF && qb < qi; ++qb) {
                const int fills = (qi - qb + C::NQBUF - 1) / C::NQBUF;
                mbar_drain(q_full(qb), uint32_t((fills - 1) & 1), p.wait_limit, p.stream_slot);
            }
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int it = 0, qi = 0;
            int npv0 = 0, npv1 = 0;   // PV MMAs issued per tile (all items)
            int nep0 = 0, nep1 = 0;   // items processed per tile (= epilogues owed)
            int qbuf = 0;   // Q buffer of the current item
            auto issue_s = [&](int t, int stage, int qb) {
                const SDesc qd = sdesc_sw128_w(sQ + (qb * C::NQ + t) * C::TILE, 16, 1024);
                const SDesc kd = sdesc_sw128_w(sKV + stage * C::TILE, 16, 1024);
                const uint32_t d = t ? tS1 : tS0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(d, qd.lo + off, qd.hi, kd.lo + off, kd.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(s_full(t));
            };
            auto issue_pv = [&](int t, int stage, bool first) {
                const SDesc vd = sdesc_sw128_w(sKV + stage * C::TILE, C::BOX, 1024);
                const uint32_t a = t ? tS1 : tS0, d = t ? tO1 : tO0;
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts_w(d, a + kk * 8, vd.lo + kk * (2048 >> 4), vd.hi, C::IDESC_PV, (!first || kk > 0) ? 1u : 0u);
                tc_commit(o_full(t));
            };
            auto wait_q = [&](int k) {   // the Q tiles of this CTA's k-th item are in place
                return mbar_wait(kRope ? q_ready(k % C::NQBUF) : q_full(k % C::NQBUF), uint32_t((k / C::NQBUF) & 1),
                                 abort_flag, p.wait_limit, kStatusTimeoutMma);
            };
            // Early start (with two Q buffers): when tile 0 has finished an item one key step before
            // tile 1, the next item's first S for tile 0 is issued before tile 1's last step, so that
            // tile 0's softmax warps start the next item instead of idling for that step.  Its Q is
            // already loaded (the other buffer), and its first K tile is the ring entry right after
            // the current item's last V tile.
            constexpr bool kEarly = C::NQBUF >= 2;
            int next_item = 0;
            bool have_next = false;   // next_item was drawn from the item ring already
            bool pre0 = false;        // S_0 of the item's first key tile was issued early, from stage pre_sk
            int pre_sk = 0;
            // S_t overwrites the columns the last PV_t read P from; both are issued by this thread,
            // and the MMAs of one thread execute in issue order, so S_t needs no wait for PV_t.
            for (;; ++qi) {
                const int item = have_next ? next_item
                                           : item_consume_thread(qi, ring, item_full0, item_empty0, abort_flag,
                                                                 p.wait_limit, kStatusTimeoutMma, ok);
                have_next = false;
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<kOffset>(p, item);
                auto act = [&](int t, int j) {
                    return t ? (g.valid1 && j >= g.jlo1 && j <= g.jhi1) : (j >= g.jlo0 && j <= g.jhi0);
                };
                qbuf = qi % C::NQBUF;
                bool first0 = true, first1 = true;
                int sk;
                if (pre0) {   // Q waited for and S_0(jbeg) issued at the end of the previous item
                    sk = pre_sk;
                    ++it;
                    pre0 = false;
                    tc_fence_after();
                    if (act(1, g.jbeg)) issue_s(1, sk, qbuf);
                } else {
                    if (!(ok = wait_q(qi))) break;
                    sk = it % C::NSTAGE;
                    ok = mbar_wait(kv_full(sk), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    ++it;
                    if (!ok) break;
                    tc_fence_after();
                    if (act(0, g.jbeg)) issue_s(0, sk, qbuf);
                    if (act(1, g.jbeg)) issue_s(1, sk, qbuf);
                }
                for (int j = g.jbeg; j <= g.jend && ok; ++j) {
                    const int sv = it % C::NSTAGE;
                    ok = mbar_wait(kv_full(sv), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    ++it;
                    if (!ok) break;
                    const bool more = j + 1 <= g.jend;
                    int sk_next = 0;
                    if (more) {
                        sk_next = it % C::NSTAGE;
                        ok = mbar_wait(kv_full(sk_next), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit,
                                       kStatusTimeoutMma);
                        ++it;
                        if (!ok) break;
                    }
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!ok) break;
                        int& npv = t ? npv1 : npv0;
                        bool& first = t ? first1 : first0;
                        if (act(t, j)) {
                            ok = mbar_wait(p_full(t), uint32_t(npv & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
                            if (!ok) break;
                            if (first) {
                                // O_t is overwritten: the previous item's epilogue must have read it.
                                const int nep = t ? nep1 : nep0;
                                if (nep > 0) {
                                    ok = mbar_wait(o_free(t), uint32_t((nep - 1) & 1), abort_flag, p.wait_limit,
                                                   kStatusTimeoutMma);
                                    if (!ok) break;
                                }
                            }
                            tc_fence_after();
                            issue_pv(t, sv, first);
                            first = false;
                            ++npv;
                        }
                        if (more && act(t, j + 1)) issue_s(t, sk_next, qbuf);
                    }
                    // K_j (read by the S MMAs issued one step earlier) and V_j are free once the
                    // MMAs issued so far complete.
                    tc_commit(kv_empty(sk));
                    tc_commit(kv_empty(sv));
                    sk = sk_next;
                    if (kEarly && ok && j + 1 == g.jend && !act(0, g.jend)) {
                        // Tile 0 is done with this item; in use now: K_jend (S_1 issued), V_jend and
                        // the next item's first K, loading behind it (ring index it + 1).
                        next_item = item_consume_thread(qi + 1, ring, item_full0, item_empty0, abort_flag,
                                                        p.wait_limit, kStatusTimeoutMma, ok);
                        have_next = true;
                        if (ok && next_item < p.n_items && (ok = wait_q(qi + 1))) {
                            pre_sk = (it + 1) % C::NSTAGE;
                            ok = mbar_wait(kv_full(pre_sk), ((it + 1) / C::NSTAGE) & 1, abort_flag, p.wait_limit,
                                           kStatusTimeoutMma);
                            if (ok) {
                                tc_fence_after();
                                issue_s(0, pre_sk, (qi + 1) % C::NQBUF);   // tile 0 is active at jbeg
                                pre0 = true;
                            }
                        }
                    }
                }
                tc_commit(q_empty(qbuf));   // every S MMA of this item has been issued
                ++nep0;
                if (g.valid1) ++nep1;
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else if (kRope && warp >= 10) {
        // --------------------- Q prologue: rotary embedding + QK norm in shared memory ---------------------
        // Thread pt takes chunk pair j of a row: the 16-byte chunk j (elements 8j .. 8j+7) and chunk
        // j + D/16 (their rotation partners, D/2 elements later), in the 128-byte-swizzled tile layout
        // of the TMA load; the D/16 threads of a row reduce its sum of squares with shuffles.
        constexpr int TPR = D / 16;                  // threads per row
        constexpr int RPI = 64 / TPR;                // rows per pass of the 64 threads
        const int pt = threadIdx.x - C::THREADS;
        const int j = pt % TPR, rsub = pt / TPR;
        const unsigned rmask = ((1u << TPR) - 1u) << ((threadIdx.x & 31) & ~(TPR - 1));
        bool ok = true;
        for (int qi = 0;; ++qi) {
            const int item = item_consume_warp(qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutEpilogue, ok);
            if (!ok || item >= p.n_items) break;
            const FwdItem g = fwd_item<kOffset>(p, item);
            const int qb = qi % C::NQBUF;
            ok = __all_sync(0xffffffffu, mbar_wait(q_full(qb), uint32_t((qi / C::NQBUF) & 1), abort_flag,
                                                   p.wait_limit, kStatusTimeoutEpilogue));
            if (!ok) break;
            const int ntile = g.valid1 ? 2 : 1;
            for (int t = 0; t < ntile; ++t) {
                const uint32_t tb = sQ + (qb * C::NQ + t) * C::TILE;
#pragma unroll 4
                for (int r0 = 0; r0 < C::BM; r0 += RPI) {
                    const int r = r0 + rsub;
                    const long long qrow = g.q0 + t * C::BM + r;
                    const long long pos = g.L + qrow;
                    if (qrow >= p.T) continue;                 // zero rows past T: nothing to rotate
                    if (pos >= p.max_pos) {                    // no table row: left as is, and reported
                        if (j == 0) report_status(p.stream_slot, kStatusPositionRange);
                        continue;
                    }
                    const int j2 = j + TPR;
                    const uint32_t a1 = tb + (j / 8) * C::BOX + r * 128 + (((j % 8) ^ (r & 7)) * 16);
                    const uint32_t a2 = tb + (j2 / 8) * C::BOX + r * 128 + (((j2 % 8) ^ (r & 7)) * 16);
                    uint4 u1, u2;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(u1.x), "=r"(u1.y), "=r"(u1.z), "=r"(u1.w) : "r"(a1));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(u2.x), "=r"(u2.y), "=r"(u2.z), "=r"(u2.w) : "r"(a2));
                    const float* crow = p.rope_cos + size_t(pos) * (D / 2) + 8 * j;
                    const float* srow = p.rope_sin + size_t(pos) * (D / 2) + 8 * j;
                    const float4 c0 = *reinterpret_cast<const float4*>(crow), c1 = *reinterpret_cast<const float4*>(crow + 4);
                    const float4 s0 = *reinterpret_cast<const float4*>(srow), s1 = *reinterpret_cast<const float4*>(srow + 4);
                    const float co[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    const float si[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                    float x1[8], x2[8];
                    bf16x8_unpack(u1, x1);
                    bf16x8_unpack(u2, x2);
                    float ss = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {   // r1 = x1 cos - x2 sin,  r2 = x1 sin + x2 cos
                        const float r1 = fmaf(x1[i], co[i], -x2[i] * si[i]);
                        const float r2 = fmaf(x1[i], si[i], x2[i] * co[i]);
                        x1[i] = r1;
                        x2[i] = r2;
                        ss = fmaf(r1, r1, ss);
                        ss = fmaf(r2, r2, ss);
                    }
#pragma unroll
                    for (int off = TPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(rmask, ss, off);
                    const float ms = ss * (1.f / D) + p.eps;
                    const float inv = ms > 0.f ? rsqrtf(ms) : 0.f;   // an all-zero row with eps = 0 stays zero
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        x1[i] *= inv;
                        x2[i] *= inv;
                    }
                    u1 = bf16x8_pack(x1);
                    u2 = bf16x8_pack(x2);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a1), "r"(u1.x), "r"(u1.y), "r"(u1.z),
                                 "r"(u1.w) : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a2), "r"(u2.x), "r"(u2.y), "r"(u2.z),
                                 "r"(u2.w) : "memory");
                }
            }
            fence_proxy_async_smem();   // the tensor core and the TMA store read the tile through the async proxy
            mbar_arrive(q_ready(qb));
            if (p.store_qrot) {
                named_barrier_sync(2, 64);   // every prologue thread's writes are fenced
                if (pt == 0) {
                    for (int t = 0; t < ntile; ++t)
                        for (int x = 0; x < C::NBOX; ++x)
                            tma_store_4d(&tm_qr, sQ + (qb * C::NQ + t) * C::TILE + x * C::BOX, x * 64, g.h,
                                         int(g.q0) + t * C::BM, g.b);
                    bulk_commit_group();
                    bulk_wait_group_read0();   // the buffer may be refilled once the store has read it
                }
            }
            if (pt == 0) mbar_arrive(q_empty(qb));
        }
        if (pt == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // stores complete before exit
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int t = warp >> 2;
        fwd_softmax_warpgroup<D, kOffset, false>(p, t ? tS1 : tS0, t ? tO1 : tO0, s_full(t), p_full(t), o_full(t),
                                                 o_free(t), ring, item_full0, item_empty0, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Forward for windows shorter than the sequence (W < T in training, W shorter than the cache in
// chunked prefill, kOffset; no prologue).
// Same tiles, K/V ring and TMEM plan as swa_fwd_kernel, with one MMA issuer thread per query
// tile (warps 9 and 10) and the key tiles of an item walked from the last to the first: tile 1
// alone at the item's last key tile (the diagonal of its rows), both tiles on the same key tile
// through the middle, tile 0 alone at the first (the window's edge of its rows).  The issuer of
// a tile that has finished its item goes on to the next one, so tile 1 starts the next item
// while tile 0 finishes this one, instead of idling for that key step.  Each issuer walks the
// ring on its own and releases every entry once (after its MMAs that read it, or at once for a
// key tile outside its band); each query tile has its own Q buffer.  With W >= T both tiles
// start at key tile 0 and tile 0 would lead tile 1 through the item, holding twice the ring
// entries; swa_fwd_kernel (one issuer, lockstep order) serves that case.
// ---------------------------------------------------------------------------
// The other MMA issuer held the issue token through 2^27 attempts (about a second): record the
// timeout and stop (see swa_fwd_short_kernel).
__device__ __noinline__ bool token_gave_up(volatile int* abort_flag) {
    abort_flag[0] = 1;
    report_status(abort_flag[1], kStatusTimeoutMma);
    return false;
}

template <int D>
struct FwdShortCfg : FwdCfg<D> {
    // kv_full, kv_empty per stage; q_full, q_empty, q_ready, s_full, p_full, o_full, o_free, mma_done
    // per tile; item_full, item_empty per entry of the item ring
    static constexpr int NUM_BAR = 2 * FwdCfg<D>::NSTAGE + 8 * FwdCfg<D>::NQ + 2 * kItemRing;
    static constexpr int OFF_MISC = FwdCfg<D>::OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;
    static constexpr int THREADS = 352;   // softmax 0..7, producer 8, MMA issuers 9 and 10
    static_assert(SMEM_USED <= 232448, "shared memory");
};

template <int D, bool kOffset = false>
__global__ void __launch_bounds__(FwdShortCfg<D>::THREADS, 1)
swa_fwd_short_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdShortCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) report_status(p.stream_slot, kStatusSmemLayout);
        return;
    }
    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (C::NSTAGE + s); };
    const uint32_t bt = bar0 + 8u * (2 * C::NSTAGE);   // per-tile barriers start here
    auto q_full = [&](int t) { return bt + 8u * t; };
    auto q_empty = [&](int t) { return bt + 8u * (C::NQ + t); };
    auto s_full = [&](int t) { return bt + 8u * (3 * C::NQ + t); };
    auto p_full = [&](int t) { return bt + 8u * (4 * C::NQ + t); };
    auto o_full = [&](int t) { return bt + 8u * (5 * C::NQ + t); };
    auto o_free = [&](int t) { return bt + 8u * (6 * C::NQ + t); };
    auto mma_done = [&](int t) { return bt + 8u * (7 * C::NQ + t); };
    const uint32_t item_full0 = bt + 8u * (8 * C::NQ), item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);
    // Issue token of the two MMA issuers (0 free, 1 held): each holds it while it issues one
    // P*V + S group, so that the groups reach the tensor pipe one after the other instead of
    // interleaved, which would delay both tiles' S.
    int* mma_token = reinterpret_cast<int*>(gbase + C::OFF_MISC + 48);
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 2);   // both MMA issuers
        }
        for (int t = 0; t < C::NQ; ++t) {
            mbar_init(q_full(t), 1);
            mbar_init(q_empty(t), 1);
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_full(t), 1);
            mbar_init(o_free(t), 128);
            mbar_init(mma_done(t), 1);
        }
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 2 + 8);   // the MMA threads and the softmax warps
        }
        abort_flag[0] = 0;
        abort_flag[1] = p.stream_slot;   // read by a wait that gives up
        *mma_token = 0;
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
    const uint32_t tS0 = tmem, tS1 = tmem + 128u;
    const uint32_t tO0 = tmem + 256u, tO1 = tmem + 256u + uint32_t(D);

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        // Key tiles are walked from the last (jend) down to the first (jbeg).  Per item: Q_1 (tile 1
        // is the one active at jend), K and V of the first key tile walked, Q_0, then the remaining
        // K / V tiles.
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int it = 0;
            int nq[2] = {0, 0};   // Q tiles loaded per query tile
            bool ok = true;
            auto load_q = [&](const FwdItem& g, int t) -> bool {
                if (nq[t] > 0 && !(ok = mbar_wait(q_empty(t), uint32_t((nq[t] - 1) & 1), abort_flag, p.wait_limit,
                                                  kStatusTimeoutProducer)))
                    return false;
                mbar_arrive_expect_tx(q_full(t), C::TILE);
                for (int x = 0; x < C::NBOX; ++x)
                    tma_load_4d(sQ + t * C::TILE + x * C::BOX, &tm_q, q_full(t), x * 64, g.h, int(g.q0) + t * 128, g.b);
                ++nq[t];
                return true;
            };
            for (int qi = 0;; ++qi) {
                const int item =
                    item_produce(p.stream_slot, qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<kOffset>(p, item);
                const int tf = g.valid1 ? 1 : 0;   // the tile active at jend
                if (!load_q(g, tf)) break;
                bool q0 = tf == 0;   // tile 0's Q is issued
                for (int j = g.jend; j >= g.jbeg && ok; --j) {
                    for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
                        const int s = it % C::NSTAGE;
                        const uint32_t ph = (it / C::NSTAGE) & 1;
                        ok = mbar_wait(kv_empty(s), ph ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutProducer);
                        if (!ok) break;
                        mbar_arrive_expect_tx(kv_full(s), C::TILE);
                        const CUtensorMap* m = kv ? &tm_v : &tm_k;
                        for (int x = 0; x < C::NBOX; ++x)
                            tma_load_4d(sKV + s * C::TILE + x * C::BOX, m, kv_full(s), x * 64, g.hk, j * C::BN, g.b);
                    }
                    if (ok && !q0 && !(q0 = load_q(g, 0))) break;
                }
            }
            work_slot_finish(p.stream_slot);
            // Drain: make sure no copy is still landing when the CTA exits.
            for (int s = 0; s < C::NSTAGE && s < it; ++s) {
                const int fills = (it - s + C::NSTAGE - 1) / C::NSTAGE;
                mbar_drain(kv_full(s), uint32_t((fills - 1) & 1), p.wait_limit, p.stream_slot);
            }
            for (int t = 0; t < C::NQ; ++t)
                if (nq[t] > 0) mbar_drain(q_full(t), uint32_t((nq[t] - 1) & 1), p.wait_limit, p.stream_slot);
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------ MMA issuers, one per query tile ------------------------------
        if (lane == 0) {
            const int t = warp - 9;
            const uint32_t tS = t ? tS1 : tS0, tO = t ? tO1 : tO0;
            bool ok = true;
            int it = 0;    // ring entries passed (used or not)
            int npv = 0;   // PV MMAs issued (all items)
            int nep = 0;   // items of this tile (= epilogues owed)
            int nq = 0;    // Q tiles waited for
            auto issue_s = [&](int stage) {
                const SDesc qd = sdesc_sw128_w(sQ + t * C::TILE, 16, 1024);
                const SDesc kd = sdesc_sw128_w(sKV + stage * C::TILE, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4;
                    mma_ss_w(tS, qd.lo + off, qd.hi, kd.lo + off, kd.hi, C::IDESC_S, kk > 0);
                }
                tc_commit(s_full(t));
            };
            auto issue_pv = [&](int stage, bool first) {
                const SDesc vd = sdesc_sw128_w(sKV + stage * C::TILE, C::BOX, 1024);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts_w(tO, tS + kk * 8, vd.lo + kk * (2048 >> 4), vd.hi, C::IDESC_PV, (!first || kk > 0) ? 1u : 0u);
                tc_commit(o_full(t));
            };
            auto take = [&](int& stage) -> bool {   // the next ring entry has landed
                stage = it % C::NSTAGE;
                ok = mbar_wait(kv_full(stage), uint32_t((it / C::NSTAGE) & 1), abort_flag, p.wait_limit,
                               kStatusTimeoutMma);
                ++it;
                return ok;
            };
            auto pass = [&](int n) -> bool {   // n ring entries this tile does not read: release them
                for (int i = 0; i < n; ++i) {
                    int s;
                    if (!take(s)) return false;
                    mbar_arrive(kv_empty(s));
                }
                return true;
            };
            auto acquire = [&]() -> bool {   // the issue token, within a bounded number of attempts
                if (atomicCAS(mma_token, 0, 1) == 0) return true;
                for (uint32_t n = 0; atomicCAS(mma_token, 0, 1) != 0;)
                    if (++n > (1u << 27)) return ok = token_gave_up(abort_flag);
                return true;
            };
            auto release = [&]() { atomicExch(mma_token, 0); };
            // S_t overwrites the columns the last PV_t read P from; both are issued by this thread,
            // and the MMAs of one thread execute in issue order, so S_t needs no wait for PV_t.
            for (int qi = 0;; ++qi) {
                const int item = item_consume_thread(qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                                     kStatusTimeoutMma, ok);
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<kOffset>(p, item);
                if (t == 1 && !g.valid1) {
                    if (!pass(2 * (g.jend - g.jbeg + 1))) break;
                    continue;
                }
                const int jlo = t ? g.jlo1 : g.jlo0, jhi = t ? g.jhi1 : g.jhi0;
                if (!pass(2 * (g.jend - jhi))) break;   // key tiles above this tile's band
                if (!(ok = mbar_wait(q_full(t), uint32_t(nq & 1), abort_flag, p.wait_limit,
                                     kStatusTimeoutMma)))
                    break;
                ++nq;
                int sk;
                if (!take(sk) || !acquire()) break;
                tc_fence_after();
                issue_s(sk);
                release();
                if (jlo == jhi) tc_commit(q_empty(t));
                for (int j = jhi; j >= jlo && ok; --j) {
                    int sv, sk_next = 0;
                    const bool more = j > jlo;
                    if (!take(sv) || (more && !take(sk_next))) break;
                    if (!(ok = mbar_wait(p_full(t), uint32_t(npv & 1), abort_flag, p.wait_limit, kStatusTimeoutMma)))
                        break;
                    // O_t is overwritten by the item's first PV: the previous epilogue must have read it.
                    if (j == jhi && nep > 0 &&
                        !(ok = mbar_wait(o_free(t), uint32_t((nep - 1) & 1), abort_flag, p.wait_limit,
                                         kStatusTimeoutMma)))
                        break;
                    if (!acquire()) break;
                    tc_fence_after();
                    issue_pv(sv, j == jhi);
                    ++npv;
                    if (more) {
                        issue_s(sk_next);
                        if (j - 1 == jlo) tc_commit(q_empty(t));   // the item's last S of this tile
                    }
                    release();
                    // K_j (read by the S MMA issued one step earlier) and V_j are free once this
                    // thread's MMAs issued so far complete.
                    tc_commit(kv_empty(sk));
                    tc_commit(kv_empty(sv));
                    sk = sk_next;
                }
                if (!ok) break;
                if (!pass(2 * (jlo - g.jbeg))) break;   // key tiles below this tile's band
                ++nep;
            }
            tc_commit(mma_done(t));
            mbar_wait(mma_done(t), 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else if (warp < 8) {
        // ------------------------------ softmax warpgroups ------------------------------
        const int t = warp >> 2;
        fwd_softmax_warpgroup<D, kOffset, true>(p, t ? tS1 : tS0, t ? tO1 : tO0, s_full(t), p_full(t), o_full(t),
                                              o_free(t), ring, item_full0, item_empty0, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Chunked prefill, append step: a chunk of Tn tokens' K and V goes to cache slots
// cache_len[b] + len_off .. cache_len[b] + len_off + Tn - 1 of each sequence, and with tail > 0
// the slots after it up to the end of that 128-slot tile are zeroed: they hold no token, and the
// forward's last key tile reads them (their scores are masked, and zero V rows keep P*V finite
// whatever the slots held).  Slots at or beyond cap are not written; a chunk that needs them
// sets kStatusCacheOverflow.  kRope: each key is rotated and normalised at its position (its
// slot) on the way in (rope.cuh).
// One thread per 16 bytes of a (slot, K/V head) row; a row's threads are consecutive lanes.
// ---------------------------------------------------------------------------
template <int D, bool kRope>
__global__ void __launch_bounds__(256) swa_append_kernel(const __nv_bfloat16* __restrict__ k_new,
                                                         const __nv_bfloat16* __restrict__ v_new,
                                                         __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
                                                         const int* __restrict__ cache_len, int B, int Tn, int cap,
                                                         int Hkv, int len_off, int tail, const float* __restrict__ cs,
                                                         const float* __restrict__ sn, int max_pos, float eps,
                                                         int stream_slot) {
    constexpr int CPR = D / 8;   // 16-byte chunks per head row
    const int span = Tn + tail;  // chunk rows plus the largest zeroed tail
    const long long total = (long long)B * span * Hkv * CPR;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const unsigned mask = rope_group_mask<D>();
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int c = int(e % CPR);
        const long long r = e / CPR;
        const int hk = int(r % Hkv);
        const int t = int((r / Hkv) % span);
        const int b = int(r / ((long long)Hkv * span));
        const long long L0 = (long long)cache_len[b] + len_off;
        if (L0 < 0 && len_off < 0) continue;   // decode of an empty sequence: no slot for the token
        const long long L = L0 < 0 ? 0 : L0;
        const long long slot = L + t;
        const long long tile_end = (L + Tn + 127) / 128 * 128;
        // every branch below is uniform over the row's threads (it depends on b, t, hk only)
        if (t >= Tn && slot >= tile_end) continue;
        if (slot >= cap) {
            if (t < Tn) report_status(stream_slot, kStatusCacheOverflow);
            continue;
        }
        const size_t dst = ((size_t(b) * cap + size_t(slot)) * Hkv + hk) * D + c * 8;
        uint4 kw = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
        if (t < Tn) {
            const size_t src = ((size_t(b) * Tn + t) * Hkv + hk) * D + c * 8;
            kw = *reinterpret_cast<const uint4*>(k_new + src);
            vw = *reinterpret_cast<const uint4*>(v_new + src);
            if (kRope) {
                if (slot >= max_pos) {
                    report_status(stream_slot, kStatusPositionRange);
                    continue;
                }
                float f[8];
                bf16x8_unpack(kw, f);
                rope_qknorm8<D>(f, c, cs + slot * (D / 2), sn + slot * (D / 2), eps, mask);
                kw = bf16x8_pack(f);
            }
        }
        *reinterpret_cast<uint4*>(kc + dst) = kw;
        *reinterpret_cast<uint4*>(vc + dst) = vw;
    }
}

}  // namespace swa
