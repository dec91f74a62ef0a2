// fwd_fp8.cuh -- FP8 (E4M3) forward of causal sliding-window attention: O and logsumexp.
//
// The pages name FP8 only for linear layers (apidog guide "Train your own ChatGPT", section 3,
// mixed precision: --fp8 on H100 and Blackwell); the attention reading here: q, k, v are OCP E4M3
// values with one fp32 descale factor per (sequence, head), the real operand being value *
// descale, and the operation is the plain windowed attention of fwd.cuh on those real operands
// (window: query i attends to keys j in (i - W, i]).
//
// Same persistent structure as the bf16 forward (one CTA per SM, items = two 128-row query tiles
// of one head, head-major, drawn from a launch-wide counter; warp 8 TMA producer, warp 9 MMA
// issuer, warps 0..7 two softmax warpgroups), with 8-bit tiles throughout:
//   S_t = Q_t K_j^T      tcgen05.mma kind::f8f6f4, e4m3 x e4m3 -> fp32 in TMEM, both operands
//                        K-major in shared memory (128-byte rows, 128-byte swizzle)
//   P_t                  exp2 of the scaled scores (scale * dq * dk folded into one factor),
//                        rounded to e4m3 into a K-major shared-memory tile
//   O_t += P_t V_j       kind::f8f6f4 with V_j^T as a K-major operand: the host transposes V once
//                        per call into the workspace ([B, Hkv, D, Tp], keys contiguous)
//   O = O * dv / l       in the epilogue (l sums the unrounded P, so the e4m3 rounding of P only
//                        perturbs the weights of the average)
// P <= 2^8 under the lazy rescale (threshold 2^8), inside e4m3's range (448).  D = 128 only.
#pragma once

#include "fwd.cuh"
#include "sm100.cuh"

namespace swa {

struct Fp8Cfg {
    static constexpr int D = 128;
    static constexpr int BM = 128, BN = 128, NQ = 2;
    static constexpr int TILE = 128 * 128;              // bytes of a 128 x 128 e4m3 tile (one TMA box)
    static constexpr int NSTAGE = 8;                    // K / V^T ring
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = NQ * TILE;
    static constexpr int OFF_KV = 2 * NQ * TILE;
    static constexpr int OFF_BAR = OFF_KV + NSTAGE * TILE;
    // kv_full, kv_empty per stage; q_full, q_empty; s_full, p_full, o_full, o_free per tile;
    // mma_done; item_full, item_empty per ring entry
    static constexpr int NUM_BAR = 2 * NSTAGE + 2 + 4 * NQ + 1 + 2 * kItemRing;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    static constexpr int SMEM = SMEM_USED + 1024;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;           // S0 | S1 | O0 | O1
    // kind::f8f6f4 instruction descriptor: D f32 (1 << 4); A, B formats E4M3 (0); both K-major
    static constexpr uint32_t IDESC = (1u << 4) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static_assert(SMEM <= 232448, "shared memory");
};

struct Fp8Params {
    __nv_bfloat16* o;       // [B, T, H, D]
    float* lse;             // [B, H, T]
    const float* dq;        // [B, H] descales
    const float* dk;        // [B, Hkv]
    const float* dv;        // [B, Hkv]
    int B, T, H, G;         // G query heads per K/V head
    long long W;
    float scale_log2;       // softmax scale * log2(e); times dq * dk per item
    int n_qblk, n_items;
    int stream_slot;
    long long wait_limit;
};

// D[tmem] (+)= A[smem desc] * B[smem desc]^T   (kind::f8f6f4, fp32 accumulate)
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four fp32 -> four e4m3 bytes (round to nearest even, saturating), element 0 in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));   // a -> low byte
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
    return uint32_t(lo) | (uint32_t(hi) << 16);
}

// V [B, T, Hkv, 128] e4m3 -> V^T [B, Hkv, 128, Tp] (keys contiguous, keys T..Tp-1 zero), so that
// the P V product reads V as a K-major operand.  One block per (64-key run, K/V head, sequence):
// 64 x 128 bytes through shared memory.
__global__ void __launch_bounds__(256) swa_fp8_transpose_v_kernel(const uint8_t* __restrict__ v,
                                                                   uint8_t* __restrict__ vt, int T, int Hkv,
                                                                   int Tp) {
    __shared__ uint8_t tile[64][128 + 16];
    const int t0 = blockIdx.x * 64, hk = blockIdx.y, b = blockIdx.z;
    for (int e = threadIdx.x; e < 64 * 8; e += blockDim.x) {   // 16-byte pieces of 64 key rows
        const int kr = e / 8, c = e % 8;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (t0 + kr < T) w = *reinterpret_cast<const uint4*>(v + ((size_t(b) * T + t0 + kr) * Hkv + hk) * 128 + c * 16);
        *reinterpret_cast<uint4*>(&tile[kr][c * 16]) = w;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 128 * 4; e += blockDim.x) {  // 16 keys of one d row per piece
        const int d = e / 4, c = e % 4;
        if (t0 + c * 16 >= Tp) continue;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = uint32_t(tile[c * 16 + 4 * i][d]) | (uint32_t(tile[c * 16 + 4 * i + 1][d]) << 8) |
                   (uint32_t(tile[c * 16 + 4 * i + 2][d]) << 16) | (uint32_t(tile[c * 16 + 4 * i + 3][d]) << 24);
        *reinterpret_cast<uint4*>(vt + ((size_t(b) * Hkv + hk) * 128 + d) * Tp + t0 + c * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void __launch_bounds__(Fp8Cfg::THREADS, 1)
swa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_vt, const Fp8Params p) {
    using C = Fp8Cfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    if (int(base - raw) + C::SMEM_USED > C::SMEM) {
        if (threadIdx.x == 0) report_status(p.stream_slot, kStatusSmemLayout);
        return;
    }
    const uint32_t sQ = base + C::OFF_Q, sP = base + C::OFF_P, sKV = base + C::OFF_KV;
    const uint32_t bar0 = base + C::OFF_BAR;
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (C::NSTAGE + s); };
    const uint32_t q_full = bar0 + 8u * (2 * C::NSTAGE), q_empty = q_full + 8u;
    const uint32_t bt = q_empty + 8u;
    auto s_full = [&](int t) { return bt + 8u * t; };
    auto p_full = [&](int t) { return bt + 8u * (C::NQ + t); };
    auto o_full = [&](int t) { return bt + 8u * (2 * C::NQ + t); };
    auto o_free = [&](int t) { return bt + 8u * (3 * C::NQ + t); };
    const uint32_t mma_done = bt + 8u * (4 * C::NQ);
    const uint32_t item_full0 = mma_done + 8u, item_empty0 = item_full0 + 8u * kItemRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 16);
    volatile int* ring = reinterpret_cast<volatile int*>(gbase + C::OFF_MISC + 32);

    // Item geometry: the bf16 forward's (query block of 256 rows, head-major, latest first).
    FwdParams ip{};
    ip.B = p.B;
    ip.T = p.T;
    ip.H = p.H;
    ip.G = p.G;
    ip.W = p.W;
    ip.n_qblk = p.n_qblk;
    const int T = p.T;
    const long long W = p.W;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int t = 0; t < C::NQ; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_full(t), 1);
            mbar_init(o_free(t), 128);
        }
        mbar_init(mma_done, 1);
        for (int e = 0; e < kItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, 1 + 8);
        }
        abort_flag[0] = 0;
        abort_flag[1] = p.stream_slot;
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
    const uint32_t tS0 = tmem, tS1 = tmem + 128u, tO0 = tmem + 256u, tO1 = tmem + 384u;

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_vt);
            int it = 0, qi = 0;
            bool ok = true;
            for (;; ++qi) {
                const int item =
                    item_produce(p.stream_slot, qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit, ok);
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<false>(ip, item);
                if (qi > 0 && !(ok = mbar_wait(q_empty, uint32_t((qi - 1) & 1), abort_flag, p.wait_limit,
                                               kStatusTimeoutProducer)))
                    break;
                mbar_arrive_expect_tx(q_full, (g.valid1 ? 2 : 1) * C::TILE);
                for (int t = 0; t < (g.valid1 ? 2 : 1); ++t)
                    tma_load_4d(sQ + t * C::TILE, &tm_q, q_full, 0, g.h, int(g.q0) + t * 128, g.b);
                for (int j = g.jbeg; j <= g.jend && ok; ++j) {
                    for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
                        const int s = it % C::NSTAGE;
                        ok = mbar_wait(kv_empty(s), ((it / C::NSTAGE) & 1) ^ 1u, abort_flag, p.wait_limit,
                                       kStatusTimeoutProducer);
                        if (!ok) break;
                        mbar_arrive_expect_tx(kv_full(s), C::TILE);
                        if (kv == 0)
                            tma_load_4d(sKV + s * C::TILE, &tm_k, kv_full(s), 0, g.hk, j * C::BN, g.b);
                        else   // V^T tile: 128 keys (x) of the 128 head-dim rows
                            tma_load_4d(sKV + s * C::TILE, &tm_vt, kv_full(s), j * C::BN, 0, g.hk, g.b);
                    }
                }
            }
            work_slot_finish(p.stream_slot);
            for (int s = 0; s < C::NSTAGE && s < it; ++s)
                mbar_drain(kv_full(s), uint32_t(((it - s + C::NSTAGE - 1) / C::NSTAGE - 1) & 1), p.wait_limit,
                           p.stream_slot);
            if (qi > 0) mbar_drain(q_full, uint32_t((qi - 1) & 1), p.wait_limit, p.stream_slot);
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int it = 0, qi = 0;
            int npv0 = 0, npv1 = 0, nep0 = 0, nep1 = 0;
            // K-major 128-byte rows in 128-byte swizzle: K steps of 32 elements are 32 bytes apart.
            auto issue_s = [&](int t, int stage) {
                const uint32_t qa = sQ + t * C::TILE, ka = sKV + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    mma_ss_f8(t ? tS1 : tS0, sdesc_sw128(qa + kk * 32, 16, 1024), sdesc_sw128(ka + kk * 32, 16, 1024),
                              C::IDESC, kk > 0);
                tc_commit(s_full(t));
            };
            auto issue_pv = [&](int t, int stage, bool first) {
                const uint32_t pa = sP + t * C::TILE, va = sKV + stage * C::TILE;
#pragma unroll
                for (int kk = 0; kk < C::BN / 32; ++kk)
                    mma_ss_f8(t ? tO1 : tO0, sdesc_sw128(pa + kk * 32, 16, 1024), sdesc_sw128(va + kk * 32, 16, 1024),
                              C::IDESC, (!first || kk > 0) ? 1u : 0u);
                tc_commit(o_full(t));
            };
            for (;; ++qi) {
                const int item = item_consume_thread(qi, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                                     kStatusTimeoutMma, ok);
                if (!ok || item >= p.n_items) break;
                const FwdItem g = fwd_item<false>(ip, item);
                auto act = [&](int t, int j) {
                    return t ? (g.valid1 && j >= g.jlo1 && j <= g.jhi1) : (j >= g.jlo0 && j <= g.jhi0);
                };
                if (!(ok = mbar_wait(q_full, uint32_t(qi & 1), abort_flag, p.wait_limit, kStatusTimeoutMma))) break;
                bool first0 = true, first1 = true;
                int sk = it % C::NSTAGE;
                ok = mbar_wait(kv_full(sk), (it / C::NSTAGE) & 1, abort_flag, p.wait_limit, kStatusTimeoutMma);
                ++it;
                if (!ok) break;
                tc_fence_after();
                if (act(0, g.jbeg)) issue_s(0, sk);
                if (act(1, g.jbeg)) issue_s(1, sk);
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
                                const int nep = t ? nep1 : nep0;
                                if (nep > 0 && !(ok = mbar_wait(o_free(t), uint32_t((nep - 1) & 1), abort_flag,
                                                                 p.wait_limit, kStatusTimeoutMma)))
                                    break;
                            }
                            tc_fence_after();
                            issue_pv(t, sv, first);
                            first = false;
                            ++npv;
                        }
                        // S_t(j+1) completes after PV_t(j) (one thread's MMAs run in issue order), so
                        // the softmax warps see P_t(j) read before they write P_t(j+1).
                        if (more && act(t, j + 1)) issue_s(t, sk_next);
                    }
                    tc_commit(kv_empty(sk));
                    tc_commit(kv_empty(sv));
                    sk = sk_next;
                }
                tc_commit(q_empty);
                ++nep0;
                if (g.valid1) ++nep1;
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, abort_flag, p.wait_limit, kStatusTimeoutMma);
        }
    } else {
        // ------------------------------ softmax warpgroups ------------------------------
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        const uint32_t tS = (t ? tS1 : tS0) + lane_off, tO = (t ? tO1 : tO0) + lane_off;
        const uint32_t prow = sP + t * C::TILE + row * 128;   // this row of the P tile (128 keys, 1 byte each)
        int ns = 0;
        bool ok = true;
        for (int k = 0;; ++k) {
            const int item = item_consume_warp(k, ring, item_full0, item_empty0, abort_flag, p.wait_limit,
                                               kStatusTimeoutSoftmax, ok);
            if (!ok || item >= p.n_items) break;
            const FwdItem g = fwd_item<false>(ip, item);
            if (t == 1 && !g.valid1) continue;
            const float sl2 = p.scale_log2 * p.dq[size_t(g.b) * p.H + g.h] * p.dk[size_t(g.b) * (p.H / p.G) + g.hk];
            const long long qt0 = g.q0 + t * 128;
            const long long q = qt0 + row;
            const int jlo = t ? g.jlo1 : g.jlo0, jhi = t ? g.jhi1 : g.jhi0;
            float m_run = -INFINITY, l_run = 0.f;
            int nloc = 0;
            for (int j = jlo; j <= jhi && ok; ++j, ++ns, ++nloc) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait(s_full(t), uint32_t(ns & 1), abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
                if (!ok) break;
                tc_fence_after();
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
                const long long k0 = (long long)j * C::BN;
                const bool full = (k0 + C::BN - 1 <= qt0) && (k0 > qt0 + C::BM - 1 - W);
                if (!full) {
                    const int chi = int(imin_ll(imax_ll(q - k0, -1), C::BN));
                    const int clo = int(imin_ll(imax_ll(q - W + 1 - k0, 0), C::BN + 1));
#pragma unroll
                    for (int c = 0; c < C::BN; ++c) s[c] = (c >= clo && c <= chi) ? s[c] : -INFINITY;
                }
                float mp[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
                for (int c = 8; c < C::BN; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
                const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                       fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
                const float m_tile = mx * sl2;
                const float m_new = fmaxf(m_run, m_tile);
                const bool warp_need = __any_sync(0xffffffffu, m_new > m_run + 8.0f);
                const float m_use = warp_need ? m_new : m_run;
                const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
                const float alpha = (m_use == -INFINITY) ? 1.f : ex2_approx(m_run - m_use);
                float sp[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) sp[u] = 0.f;
                // P in e4m3, 16 keys (one 16-byte piece of the swizzled row) at a time
#pragma unroll
                for (int c = 0; c < C::BN / 16; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float e[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            e[u] = ex2_approx(fmaf(s[c * 16 + 4 * i + u], sl2, -m_sub));
                            sp[(4 * i + u) & 7] += e[u];
                        }
                        w[i] = pack_e4m3x4(e[0], e[1], e[2], e[3]);
                    }
                    const uint32_t dst = prow + ((c ^ (row & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w[0]), "r"(w[1]),
                                 "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                fence_proxy_async_smem();   // the P tile is read by the tensor core (async proxy)
                const float rowsum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
                l_run = l_run * alpha + rowsum;
                if (warp_need && nloc > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(o_full(t), uint32_t((ns - 1) & 1), abort_flag,
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
                mbar_arrive(p_full(t));
            }
            if (!ok || nloc == 0) break;
            ok = __all_sync(0xffffffffu, mbar_wait(o_full(t), uint32_t((ns - 1) & 1), abort_flag, p.wait_limit,
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
            mbar_arrive(o_free(t));
            if (q < T) {
                const float mul = p.dv[size_t(g.b) * (p.H / p.G) + g.hk] / l_run;
                __nv_bfloat16* orow = p.o + ((size_t(g.b) * T + size_t(q)) * p.H + g.h) * D;
                store_row_bf16<D>(orow, ov, mul);
                p.lse[(size_t(g.b) * p.H + g.h) * T + q] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace swa
