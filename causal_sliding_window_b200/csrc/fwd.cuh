// fwd.cuh -- forward kernel: O and logsumexp of causal sliding-window attention.
//
// The operation is the one nanochat's GPT calls once per layer,
// flash_attn_func(q, k, v, causal=True, window_size=W) (apidog guide "Train
// your own ChatGPT", section 5 "Flash Attention unification"), with the
// per-layer short/long windows of the "SSSL" pattern (same guide, section 1
// "GPT model", architecture features).  Query i attends to keys
// j in (i - W, i]; W >= T is full causal.
//
// One CTA owns two 128-row query tiles of one (b, h) and walks the key/value
// tiles that intersect the band of either tile:
//   warp 8      TMA producer: Q tiles once, then K_j, V_j into a ring of stages
//   warp 9      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM, then
//               O_t += P_t V_j with P_t read from TMEM
//   warps 0..7  two softmax warpgroups, one per query tile; thread = row.
//               Online softmax in the exp2 domain, P written back to TMEM as
//               bf16 over the first half of S_t's columns, O rescaled in TMEM
//               only when a warp's running max grows by more than 2^8.
// Key tiles entirely outside the band are never loaded; only tiles that cut
// the diagonal or the window's left edge are masked element by element.
#pragma once

#include "sm100.cuh"

namespace swa {

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                  // query rows per tile (one MMA M)
    static constexpr int BN = 128;                  // key rows per tile
    static constexpr int NQ = 2;                    // query tiles per CTA
    static constexpr int TILE = 128 * D * 2;        // bytes of a 128 x D bf16 tile
    static constexpr int BOX = 128 * 64 * 2;        // one TMA box: 128 rows x 64 columns
    static constexpr int NBOX = D / 64;
    static constexpr int NSTAGE = D == 128 ? 5 : 8; // K/V ring (a stage holds one K or one V tile)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = NQ * TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    static constexpr int NUM_BAR = 2 * NSTAGE + 4 * NQ + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    // Up to 1 KB of slack to align the tile region to 1024 bytes, within the per-block limit;
    // the kernel checks at run time that the aligned layout fits what it was given.
    static constexpr int SMEM = SMEM_USED + 1024 <= 232448 ? SMEM_USED + 1024 : 232448;   // + slack for 1024-byte alignment
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;      // S0 | S1 | O0 | O1
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(SMEM_USED <= 232448, "shared memory");
};

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    int B, T, H;
    long long W;
    float scale_log2;     // softmax scale * log2(e)
    int n_qblk;           // ceil(T / 256)
    long long wait_limit; // clock cycles before a wait gives up
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {   // uniform across the CTA: nothing started yet
        if (threadIdx.x == 0) atomicOr(&g_attn_status, kStatusSmemLayout);
        return;
    }

    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    // barrier indices
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (C::NSTAGE + s); };
    auto q_full = [&](int t) { return bar0 + 8u * (2 * C::NSTAGE + t); };
    auto s_full = [&](int t) { return bar0 + 8u * (2 * C::NSTAGE + C::NQ + t); };
    auto p_full = [&](int t) { return bar0 + 8u * (2 * C::NSTAGE + 2 * C::NQ + t); };
    auto o_full = [&](int t) { return bar0 + 8u * (2 * C::NSTAGE + 3 * C::NQ + t); };
    const uint32_t mma_done = bar0 + 8u * (2 * C::NSTAGE + 4 * C::NQ);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);

    // ---- which (query block, b, h) this CTA owns; heaviest query blocks first ----
    const int BH = p.B * p.H;
    const int qblk = p.n_qblk - 1 - int(blockIdx.x / BH);
    const int bh = int(blockIdx.x % BH);
    const int b = bh / p.H, h = bh % p.H;
    const int T = p.T;
    const long long W = p.W;

    long long q0[C::NQ];
    bool tvalid[C::NQ];
    int jlo[C::NQ], jhi[C::NQ];
#pragma unroll
    for (int t = 0; t < C::NQ; ++t) {
        q0[t] = (long long)qblk * (C::BM * C::NQ) + t * C::BM;
        tvalid[t] = q0[t] < T;
        jlo[t] = int(imax_ll(0, q0[t] - W + 1) / C::BN);
        jhi[t] = int(imin_ll(q0[t] + C::BM - 1, T - 1) / C::BN);
    }
    const int nt = tvalid[1] ? 2 : 1;
    const int jbeg = jlo[0];
    const int jend = jhi[nt - 1];

    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int t = 0; t < C::NQ; ++t) {
            mbar_init(q_full(t), 1);
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_full(t), 1);
        }
        mbar_init(mma_done, 1);
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
    const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
    const uint32_t tO[2] = {tmem + 256u, tmem + 256u + uint32_t(D)};

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            for (int t = 0; t < nt; ++t) {
                mbar_arrive_expect_tx(q_full(t), C::TILE);
                for (int x = 0; x < C::NBOX; ++x)
                    tma_load_4d(sQ + t * C::TILE + x * C::BOX, &tm_q, q_full(t), x * 64, h, int(q0[t]), b);
            }
            int it = 0;
            bool ok = true;
            for (int j = jbeg; j <= jend && ok; ++j) {
                for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
                    const int s = it % C::NSTAGE;
                    const uint32_t ph = (it / C::NSTAGE) & 1;
                    ok = mbar_wait(kv_empty(s), ph ^ 1u, abort_flag, p.wait_limit, kStatusTimeoutProducer);
                    if (!ok) break;
                    mbar_arrive_expect_tx(kv_full(s), C::TILE);
                    const CUtensorMap* m = kv ? &tm_v : &tm_k;
                    for (int x = 0; x < C::NBOX; ++x)
                        tma_load_4d(sKV + s * C::TILE + x * C::BOX, m, kv_full(s), x * 64, h, j * C::BN, b);
                }
            }
            // Drain: make sure no copy is still landing when the CTA exits.
            for (int s = 0; s < C::NSTAGE && s < it; ++s) {
                const int fills = (it - s + C::NSTAGE - 1) / C::NSTAGE;
                mbar_wait(kv_full(s), uint32_t((fills - 1) & 1), abort_flag, p.wait_limit, kStatusTimeoutProducer);
            }
            for (int t = 0; t < nt; ++t) mbar_wait(q_full(t), 0, abort_flag, p.wait_limit, kStatusTimeoutProducer);
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            for (int t = 0; t < nt && ok; ++t) ok = mbar_wait(q_full(t), 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
            int it = 0;            // ring position of the next tile to consume
            int npv[2] = {0, 0};   // PV MMAs issued per query tile
            auto issue_s = [&](int t, int stage) {
                const uint32_t qa = sQ + t * C::TILE, ka = sKV + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tS[t], sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), C::IDESC_S,
                           kk > 0);
                }
                tc_commit(s_full(t));
            };
            auto issue_pv = [&](int t, int stage) {
                const uint32_t va = sKV + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ts(tO[t], tS[t] + kk * 8, sdesc_sw128(va + kk * 2048, C::BOX, 1024), C::IDESC_PV,
                           (npv[t] > 0 || kk > 0) ? 1u : 0u);
                ++npv[t];
                tc_commit(o_full(t));
            };
            // Prologue: S_t(jbeg) for the tiles whose band starts there.
            int sk = 0;
            if (ok) {
                sk = it % C::NSTAGE;
                ok = mbar_wait(kv_full(sk), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                ++it;
                tc_fence_after();
                for (int t = 0; t < nt && ok; ++t)
                    if (jbeg >= jlo[t] && jbeg <= jhi[t]) issue_s(t, sk);
            }
            for (int j = jbeg; j <= jend && ok; ++j) {
                const int sv = it % C::NSTAGE;
                ok = mbar_wait(kv_full(sv), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                ++it;
                if (!ok) break;
                const bool more = j + 1 <= jend;
                int sk_next = 0;
                if (more) {
                    sk_next = it % C::NSTAGE;
                    ok = mbar_wait(kv_full(sk_next), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                    ++it;
                    if (!ok) break;
                }
                for (int t = 0; t < nt && ok; ++t) {
                    if (j >= jlo[t] && j <= jhi[t]) {
                        ok = mbar_wait(p_full(t), uint32_t((npv[t]) & 1), abort_flag, p.wait_limit, kStatusTimeoutMma);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(t, sv);
                    }
                    if (more && j + 1 >= jlo[t] && j + 1 <= jhi[t]) {
                        // S_t(j+1) overwrites the columns PV_t(j) reads P from: wait for it.
                        if (npv[t] > 0) {
                            ok = mbar_wait(o_full(t), uint32_t((npv[t] - 1) & 1), abort_flag, p.wait_limit,
                                           kStatusTimeoutMma);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_s(t, sk_next);
                    }
                }
                // K_{j} (consumed by the S MMAs issued one step earlier) and V_j are free once
                // the MMAs issued so far complete.
                tc_commit(kv_empty(sk));
                tc_commit(kv_empty(sv));
                sk = sk_next;
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int t = warp >> 2;            // query tile of this warpgroup
        const int quarter = warp & 3;       // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;
        const long long q = q0[t] + row;    // global query index of this thread
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        int n = 0;
        bool ok = tvalid[t];
        const bool active = tvalid[t];
        if (active) {
            for (int j = jlo[t]; j <= jhi[t] && ok; ++j, ++n) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait(s_full(t), uint32_t(n & 1), abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
                float s[C::BN];
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tS[t] + lane_off + c * 32, r);
                    tmem_ld_wait(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
                }
                // Tiles that cut the diagonal or the window's left edge: keep columns clo..chi of this
                // row (keys k0+c with q-W < k0+c <= q).  The test is uniform across the CTA.
                const long long k0 = (long long)j * C::BN;
                const bool full = (k0 + C::BN - 1 <= q0[t]) && (k0 > q0[t] + C::BM - 1 - W);
                if (!full) {
                    const int chi = int(imin_ll(imax_ll(q - k0, -1), C::BN));
                    const int clo = int(imin_ll(imax_ll(q - W + 1 - k0, 0), C::BN + 1));
#pragma unroll
                    for (int c = 0; c < C::BN; ++c) s[c] = (c >= clo && c <= chi) ? s[c] : -INFINITY;
                }
                float mx = s[0];
#pragma unroll
                for (int c = 1; c < C::BN; ++c) mx = fmaxf(mx, s[c]);
                const float m_tile = mx * sl2;
                const float m_new = fmaxf(m_run, m_tile);
                const bool need = m_new > m_run + 8.0f;
                const bool warp_need = __any_sync(0xffffffffu, need);
                const float m_use = warp_need ? m_new : m_run;
                const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
                const float alpha = (m_use == -INFINITY) ? 1.f : ex2_approx(m_run - m_use);
                float rowsum = 0.f;
#pragma unroll
                for (int c = 0; c < C::BN / 64; ++c) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float p0 = ex2_approx(fmaf(s[c * 64 + 2 * i], sl2, -m_sub));
                        const float p1 = ex2_approx(fmaf(s[c * 64 + 2 * i + 1], sl2, -m_sub));
                        rowsum += p0 + p1;
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tS[t] + lane_off + c * 32, pk);
                }
                l_run = l_run * alpha + rowsum;
                tmem_st_wait();
                if (warp_need && n > 0) {
                    // O_t holds the sum up to key tile j-1: wait for PV_t(j-1), then rescale.
                    ok = __all_sync(0xffffffffu, mbar_wait(o_full(t), uint32_t((n - 1) & 1), abort_flag,
                                                           p.wait_limit, kStatusTimeoutSoftmax));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tO[t] + lane_off + c * 32, r);
                        tmem_ld_wait(r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(tO[t] + lane_off + c * 32, r);
                    }
                    tmem_st_wait();
                }
                m_run = m_use;
                tc_fence_before();
                mbar_arrive(p_full(t));
            }
            // ---- epilogue: O = O / l, lse = ln(sum exp S) ----
            if (ok && n > 0)
                ok = __all_sync(0xffffffffu, mbar_wait(o_full(t), uint32_t((n - 1) & 1), abort_flag, p.wait_limit,
                                                       kStatusTimeoutEpilogue));
            if (ok && n > 0) {
                tc_fence_after();
                const float inv_l = 1.f / l_run;
                const bool in_range = q < T;
                __nv_bfloat16* orow = p.o + ((size_t(b) * T + size_t(in_range ? q : 0)) * p.H + h) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tO[t] + lane_off + c * 32, r);
                    tmem_ld_wait(r);
                    if (in_range) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(r[v4 * 8 + 0]) * inv_l, __uint_as_float(r[v4 * 8 + 1]) * inv_l);
                            w.y = pack_bf16x2(__uint_as_float(r[v4 * 8 + 2]) * inv_l, __uint_as_float(r[v4 * 8 + 3]) * inv_l);
                            w.z = pack_bf16x2(__uint_as_float(r[v4 * 8 + 4]) * inv_l, __uint_as_float(r[v4 * 8 + 5]) * inv_l);
                            w.w = pack_bf16x2(__uint_as_float(r[v4 * 8 + 6]) * inv_l, __uint_as_float(r[v4 * 8 + 7]) * inv_l);
                            *reinterpret_cast<uint4*>(orow + c * 32 + v4 * 8) = w;
                        }
                    }
                }
                if (in_range)
                    p.lse[(size_t(b) * p.H + h) * T + q] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace swa
