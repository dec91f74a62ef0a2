// decode.cuh -- single-token decode over a KV cache, split along the cache.
//
// The inference engine keeps a per-layer K/V cache and attends the new token
// to it through flash_attn_with_kvcache (apidog guide "Train your own
// ChatGPT", section 6 "Inference engine", KV cache).  Sequence b holds
// L = cache_len[b] tokens; the new query sits at position L-1 and attends to
// slots max(0, L-W) .. L-1 of its cache.
//
// Layout: caches [B, cap, Hk, D] bf16, so one cache slot of one sequence is a
// contiguous Hk*D*2-byte row (3 KB at Hk=12, D=128).  A CTA takes a chunk of
// consecutive slots of one sequence and up to kDecodeThreads*8/D (K/V head, query subgroup)
// pairs (4 at D = 128): thread slot (pair, c) owns the 16-byte piece c of the pair's K/V head and
// serves the QPT query heads of its subgroup from it, so with grouped heads each K/V row is
// loaded once for up to QPT query heads (QPT = 1 when every query head has its own K/V head).
// The pairs of a CTA are consecutive, so its K/V reads of one slot are contiguous, coalesced,
// vectorised sweeps.  Small CTAs put more of them, and so more loads, in flight (measured: 64
// threads per CTA beat 256 by about 4% on the 12-head decode workload).  Per query head, the
// D/8 threads of a pair reduce q.k with warp shuffles and keep an online softmax (m, l) and 8
// output accumulators in registers.  Each CTA writes its partials (m, l, o) to the workspace;
// the last CTA of a (sequence, pair group) (atomic ticket) merges them:
//   M = max_c m_c,  l = sum_c 2^(m_c - M) l_c,  o = sum_c 2^(m_c - M) o_c / l.
// Slots outside the window are never read.
#pragma once

#include <cuda_bf16.h>

#include "rope.cuh"
#include "sm100.cuh"

namespace swa {

constexpr int kDecodeChunk = 128;     // cache slots per CTA, one query head per thread
constexpr int kDecodeChunkGrp = 64;   // cache slots per CTA when a thread serves several query heads
constexpr int kDecodeUnroll = 4;   // slots per batch (two batches in flight per thread)

struct DecParams {
    const __nv_bfloat16* q;        // [B,H,D]
    const __nv_bfloat16* kc;       // [B,cap,Hk,D], Hk = H / kv_group
    const __nv_bfloat16* vc;
    const int32_t* cache_len;      // [B]
    __nv_bfloat16* o;              // [B,H,D]
    float* lse;                    // [B,H] or null
    int* counters;                 // [B, pair groups], zero between calls
    float* part_ml;                // [B, nsplit_max, H, 2]
    float* part_o;                 // [B, nsplit_max, H, D]
    int B, cap, H;
    int kv_group;                  // query heads per K/V head: query head h reads cache head h / kv_group
    int nsub;                      // query-head subgroups per K/V head: ceil(kv_group / QPT)
    int chunk;                     // cache slots per CTA
    long long W;
    float scale_log2;
    int nsplit;                    // splits launched per sequence
    int nsplit_max;                // stride of the partial arrays
    // kRope: the query is rotated and normalised at its position cache_len[b] - 1 (rope.cuh), and
    // the new token's key (rotated, normalised) and value are written into that slot first
    const __nv_bfloat16* k_new;    // [B, Hk, D]
    const __nv_bfloat16* v_new;
    __nv_bfloat16* kc_out;         // the caches kc / vc, written at slot cache_len[b] - 1
    __nv_bfloat16* vc_out;
    const float* rope_cos;         // [max_pos, D/2]
    const float* rope_sin;
    int max_pos;
    float eps;
    int stream_slot;               // the launch's stream slot (status word)
};

constexpr int kDecodeThreads = 64;   // threads per CTA: D/8 per pair, so 4 pairs at D = 128 (more CTAs in flight)

template <int D>
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h2[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// Query heads per thread for kv_group query heads per K/V head: a divisor of kv_group up to 4
// where there is one, else 4 with a ragged last subgroup.
inline int decode_qpt(int kv_group) {
    if (kv_group <= 1) return 1;
    if (kv_group % 4 == 0) return 4;
    if (kv_group % 3 == 0) return 3;
    if (kv_group % 2 == 0) return 2;
    return 4;
}

template <int D, int QPT, bool kRope>
__global__ void __launch_bounds__(kDecodeThreads) swa_decode_kernel(const DecParams p) {
    constexpr int LPH = D / 8;                       // threads per (K/V head, query subgroup) pair
    constexpr int G = kDecodeThreads / LPH;          // pairs per CTA
    const int split = blockIdx.x, b = blockIdx.y, zg = blockIdx.z;
    const int H = p.H, kvg = p.kv_group;
    const int npairs = (H / kvg) * p.nsub;
    const int pr0 = zg * G;
    const int slots = min(G, npairs - pr0) * LPH;
    const int tid = threadIdx.x;
    const bool live = tid < slots;
    const int pr = pr0 + (live ? tid / LPH : 0);
    const int hk = pr / p.nsub;                      // K/V head of this thread
    const int qs = (pr % p.nsub) * QPT;              // first query head of the subgroup within the group
    const int c = tid % LPH;
    int* counter = p.counters + size_t(b) * gridDim.z + zg;
    bool hv[QPT];                                    // query head a of this thread exists
    int hq[QPT];                                     // its index (clamped for the ragged subgroup)
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        hv[a] = live && (qs + a < kvg);
        hq[a] = hk * kvg + min(qs + a, kvg - 1);
    }

    int L = p.cache_len[b];
    L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
    const long long lo_ll = (long long)L - p.W;
    const int lo = lo_ll < 0 ? 0 : int(lo_ll);
    const int start = lo + split * p.chunk;
    const int end = min(start + p.chunk, L);

    float qv[QPT][8];
    int rpos = 0;   // position of the new token (kRope); the same for every thread of the CTA
    if (kRope) {
        rpos = L - 1;
        if (rpos >= p.max_pos) {
            if (tid == 0 && split == 0) report_status(p.stream_slot, kStatusPositionRange);
            rpos = 0;
        }
        rpos = rpos < 0 ? 0 : rpos;
    }
    if (kRope && start < end && end == L && L - 1 < p.max_pos) {
        // This CTA's chunk holds the new token's slot: write the token's rotated, normalised key
        // and its value there before any load.  Other CTAs of the sequence that read the slot
        // write the same bytes themselves first, so no CTA waits for another.
        if (live) {   // uniform over a pair's threads
            const size_t src = (size_t(b) * (H / kvg) + hk) * D + c * 8;
            float f[8];
            bf16x8_to_f32<D>(*reinterpret_cast<const uint4*>(p.k_new + src), f);
            rope_qknorm8<D>(f, c, p.rope_cos + size_t(rpos) * (D / 2), p.rope_sin + size_t(rpos) * (D / 2), p.eps,
                            rope_group_mask<D>());
            const size_t dst = (size_t(b) * p.cap + size_t(L - 1)) * (size_t(H / kvg) * D) + size_t(hk) * D + c * 8;
            *reinterpret_cast<uint4*>(p.kc_out + dst) = bf16x8_pack(f);
            *reinterpret_cast<uint4*>(p.vc_out + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
        }
        __syncthreads();   // the block's loads below see the slot
    }
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        const uint4 u = hv[a] ? *reinterpret_cast<const uint4*>(p.q + (size_t(b) * H + hq[a]) * D + c * 8)
                              : make_uint4(0, 0, 0, 0);
        bf16x8_to_f32<D>(u, qv[a]);
        if (kRope) {   // every thread of the warp takes part (rows are whole groups of D/8 lanes)
            rope_qknorm8<D>(qv[a], c, p.rope_cos + size_t(rpos) * (D / 2), p.rope_sin + size_t(rpos) * (D / 2),
                            p.eps, rope_group_mask<D>());
            // a bf16 activation, as the rotated queries of prefill and training are
            bf16x8_to_f32<D>(bf16x8_pack(qv[a]), qv[a]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[a][i] *= p.scale_log2;
    }
    float m[QPT], l[QPT], acc[QPT][8];
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        m[a] = -INFINITY;
        l[a] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[a][i] = 0.f;
    }

    const size_t row_elems = size_t(H / kvg) * D;   // one cache slot: all K/V heads
    const __nv_bfloat16* kb = p.kc + size_t(b) * p.cap * row_elems + size_t(hk) * D + c * 8;
    const __nv_bfloat16* vb = p.vc + size_t(b) * p.cap * row_elems + size_t(hk) * D + c * 8;

    // Two batches of kDecodeUnroll slots are in flight: the next batch's loads are issued
    // before the current batch is consumed.
    auto load = [&](int pos, uint4 (&ku)[kDecodeUnroll], uint4 (&vu)[kDecodeUnroll]) {
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const bool in = live && (pos + u < end);
            ku[u] = in ? __ldcs(reinterpret_cast<const uint4*>(kb + size_t(pos + u) * row_elems)) : make_uint4(0, 0, 0, 0);
            vu[u] = in ? __ldcs(reinterpret_cast<const uint4*>(vb + size_t(pos + u) * row_elems)) : make_uint4(0, 0, 0, 0);
        }
    };
    auto consume = [&](int pos, const uint4 (&ku)[kDecodeUnroll], const uint4 (&vu)[kDecodeUnroll]) {
        float s[QPT][kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            float kf[8];
            bf16x8_to_f32<D>(ku[u], kf);
            float d[QPT];
#pragma unroll
            for (int a = 0; a < QPT; ++a) {
                d[a] = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) d[a] = fmaf(qv[a][i], kf[i], d[a]);
            }
#pragma unroll
            for (int off = LPH / 2; off > 0; off >>= 1)
#pragma unroll
                for (int a = 0; a < QPT; ++a) d[a] += __shfl_xor_sync(0xffffffffu, d[a], off);
#pragma unroll
            for (int a = 0; a < QPT; ++a) s[a][u] = (pos + u < end) ? d[a] : -INFINITY;
        }
        float mx[QPT];
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            mx[a] = m[a];
#pragma unroll
            for (int u = 0; u < kDecodeUnroll; ++u) mx[a] = fmaxf(mx[a], s[a][u]);
            const float alpha = ex2_approx(m[a] - mx[a]);   // m = -inf on the first batch: alpha = 0
            l[a] *= alpha;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[a][i] *= alpha;
            m[a] = mx[a];
        }
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            float vf[8];
            bf16x8_to_f32<D>(vu[u], vf);
#pragma unroll
            for (int a = 0; a < QPT; ++a) {
                const float pu = ex2_approx(s[a][u] - mx[a]);
                l[a] += pu;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[a][i] = fmaf(pu, vf[i], acc[a][i]);
            }
        }
    };
    uint4 ka[kDecodeUnroll], va[kDecodeUnroll], kn[kDecodeUnroll], vn[kDecodeUnroll];
    if (start < end) load(start, ka, va);
    for (int pos = start; pos < end; pos += 2 * kDecodeUnroll) {   // CTA-uniform trip count
        if (pos + kDecodeUnroll < end) load(pos + kDecodeUnroll, kn, vn);
        consume(pos, ka, va);
        if (pos + 2 * kDecodeUnroll < end) load(pos + 2 * kDecodeUnroll, ka, va);
        if (pos + kDecodeUnroll < end) consume(pos + kDecodeUnroll, kn, vn);
    }

    // ---- partials of this chunk ----
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        if (!hv[a]) continue;
        const size_t pidx = (size_t(b) * p.nsplit_max + split) * H + hq[a];
        float4* po = reinterpret_cast<float4*>(p.part_o + pidx * D + c * 8);
        po[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        po[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
        if (c == 0) {
            p.part_ml[2 * pidx] = m[a];
            p.part_ml[2 * pidx + 1] = l[a];
        }
    }
    __threadfence();
    __syncthreads();
    __shared__ int is_last;
    if (tid == 0) {
        const int ticket = atomicAdd(counter, 1);
        is_last = (ticket == p.nsplit - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---- last CTA of this (sequence, pair group): merge the partials of the non-empty chunks ----
    // One pass with a running maximum; the loads of MB partials of every query head of the thread
    // are in flight together (MB = 2 at 3-4 heads per thread keeps the registers of the main loop
    // in bounds).  Every used chunk holds at least one slot, so its m is finite.
    constexpr int MB = QPT >= 3 ? 2 : 4;
    const int n = L - lo;
    const int used = (n + p.chunk - 1) / p.chunk;
    float M[QPT], lsum[QPT], o8[QPT][8];
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        M[a] = -INFINITY;
        lsum[a] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) o8[a][i] = 0.f;
    }
    const size_t pbase = size_t(b) * p.nsplit_max * H;   // partial (split sp, head h) at pbase + sp * H + h
    for (int sp0 = 0; sp0 < used; sp0 += MB) {
        float ml[QPT][MB][2];
        float4 oa[QPT][MB], ob[QPT][MB];
#pragma unroll
        for (int a = 0; a < QPT; ++a)
#pragma unroll
            for (int u = 0; u < MB; ++u) {
                const bool in = hv[a] && sp0 + u < used;
                const size_t q = pbase + size_t(sp0 + u) * H + hq[a];
                ml[a][u][0] = in ? __ldcg(p.part_ml + 2 * q) : -INFINITY;
                ml[a][u][1] = in ? __ldcg(p.part_ml + 2 * q + 1) : 0.f;
                oa[a][u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8)) : make_float4(0, 0, 0, 0);
                ob[a][u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8) + 1)
                              : make_float4(0, 0, 0, 0);
            }
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            float bm = M[a];
#pragma unroll
            for (int u = 0; u < MB; ++u) bm = fmaxf(bm, ml[a][u][0]);
            if (bm == -INFINITY) continue;                 // head a not served by this thread
            const float sc = ex2_approx(M[a] - bm);        // 0 on the first batch (M = -inf)
            lsum[a] *= sc;
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[a][i] *= sc;
#pragma unroll
            for (int u = 0; u < MB; ++u) {
                const float w = ex2_approx(ml[a][u][0] - bm);   // 0 for padding entries (m = -inf)
                lsum[a] = fmaf(w, ml[a][u][1], lsum[a]);
                o8[a][0] = fmaf(w, oa[a][u].x, o8[a][0]);
                o8[a][1] = fmaf(w, oa[a][u].y, o8[a][1]);
                o8[a][2] = fmaf(w, oa[a][u].z, o8[a][2]);
                o8[a][3] = fmaf(w, oa[a][u].w, o8[a][3]);
                o8[a][4] = fmaf(w, ob[a][u].x, o8[a][4]);
                o8[a][5] = fmaf(w, ob[a][u].y, o8[a][5]);
                o8[a][6] = fmaf(w, ob[a][u].z, o8[a][6]);
                o8[a][7] = fmaf(w, ob[a][u].w, o8[a][7]);
            }
            M[a] = bm;
        }
    }
#pragma unroll
    for (int a = 0; a < QPT; ++a) {
        if (!hv[a]) continue;
        const float inv = used > 0 ? 1.f / lsum[a] : 0.f;
        uint4 w;
        w.x = pack_bf16x2(o8[a][0] * inv, o8[a][1] * inv);
        w.y = pack_bf16x2(o8[a][2] * inv, o8[a][3] * inv);
        w.z = pack_bf16x2(o8[a][4] * inv, o8[a][5] * inv);
        w.w = pack_bf16x2(o8[a][6] * inv, o8[a][7] * inv);
        *reinterpret_cast<uint4*>(p.o + (size_t(b) * H + hq[a]) * D + c * 8) = w;
        if (c == 0 && p.lse != nullptr)
            p.lse[size_t(b) * H + hq[a]] = used > 0 ? (M[a] + log2f(lsum[a])) * 0.69314718055994530942f : -INFINITY;
    }
    if (tid == 0) *counter = 0;   // ready for the next call
}

}  // namespace swa
