// decode.cuh -- single-token decode over a KV cache, split along the cache.
//
// The inference engine keeps a per-layer K/V cache and attends the new token
// to it through flash_attn_with_kvcache (apidog guide "Train your own
// ChatGPT", section 6 "Inference engine", KV cache).  Sequence b holds
// L = cache_len[b] tokens; the new query sits at position L-1 and attends to
// slots max(0, L-W) .. L-1 of its cache.
//
// Layout: caches [B, cap, Hk, D] bf16, so one cache slot of one sequence is a
// contiguous Hk*D*2-byte row (3 KB at Hk=12, D=128), and a run of slots is one
// contiguous block.
//
// Persistent and streaming: one CTA per SM draws work items from a launch-wide counter.
// An item is (chunk c of kDecodeChunk window slots, sequence b, head group g); items whose
// chunk holds no slot of the window are skipped by the draw itself, so short sequences
// cost nothing.  Warp 0 (one thread) streams the item's K and V rows (the K/V heads of the
// group) into a ring of shared-memory stages with bulk copies (cp.async.bulk), many tens of
// KB in flight per SM, while the other warps compute.  Consumer thread (pair, c) owns the
// 16-byte piece c of a (K/V head, query subgroup) pair and serves the QPT query heads of its
// subgroup from it (QPT = 1 when every query head has its own K/V head), so with grouped
// heads each K/V row is read once for up to QPT query heads.  Per query head the D/8 threads
// of a pair reduce q.k with warp shuffles and keep an online softmax (m, l) and 8 output
// accumulators in registers.  Each item's partials (m, l, o) go to the workspace; the CTA
// that finishes the last chunk of a (sequence, head group) (atomic ticket) merges them:
//   M = max_c m_c,  l = sum_c 2^(m_c - M) l_c,  o = sum_c 2^(m_c - M) o_c / l.
// Slots outside the window are never read.
#pragma once

#include <cuda_bf16.h>

#include "rope.cuh"
#include "sm100.cuh"

namespace swa {

constexpr int kDecodeChunk = 64;           // window slots per work item
// Consumer threads per CTA at most: fewer when a thread serves several query heads, so that
// its accumulators stay in registers.
__host__ __device__ constexpr int decode_max_consumers(int qpt) { return qpt == 1 ? 384 : 256; }
constexpr int kDecodeUnroll = 4;           // slots per batch of loads from shared memory
constexpr int kDecodeItemRing = 4;
// Up to this many sequences, every CTA first builds the prefix sum of the sequences' chunk counts
// in shared memory, so that item i of the launch maps straight to a chunk that holds window slots;
// larger batches enumerate every (chunk, sequence) and skip the empty ones while drawing.
constexpr int kDecodePrefixMax = 4096;

struct DecParams {
    const __nv_bfloat16* q;        // [B,H,D]
    const __nv_bfloat16* kc;       // [B,cap,Hk,D], Hk = H / kv_group
    const __nv_bfloat16* vc;
    const int32_t* cache_len;      // [B]
    __nv_bfloat16* o;              // [B,H,D]
    float* lse;                    // [B,H] or null
    int* tickets;                  // [B, ngroups], zero between calls
    float* part_ml;                // [B, nsplit_max, H, 2]
    float* part_o;                 // [B, nsplit_max, H, D]
    int B, cap, H, Hk;
    int kv_group;                  // query heads per K/V head: query head h reads cache head h / kv_group
    int nsub;                      // query-head subgroups per K/V head: ceil(kv_group / QPT)
    int gh;                        // K/V heads per head group (the last group may have fewer)
    int ngroups;
    int ss;                        // cache slots per shared-memory stage
    int nstage;                    // stages in the ring
    long long W;
    float scale_log2;
    int nsplit;                    // chunks per sequence: ceil(min(W, cap) / kDecodeChunk)
    int nsplit_max;                // stride of the partial arrays: ceil(cap / kDecodeChunk)
    int n_items;                   // nsplit * B * ngroups: items without the prefix (B > kDecodePrefixMax)
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
    int stream_slot;               // the launch's stream slot: work counter and status word
    long long wait_limit;
};

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

// Window geometry of sequence b and its chunk c.  With the prefix (pref[b] = chunks of sequences
// before b, pref[B] = all of them) item = chunk index over all sequences * ngroups + group;
// without it, item = (c * B + b) * ngroups + g over every possible chunk.
struct DecItem {
    int b, c, g;
    int L, lo, start, end;
};
__device__ __forceinline__ DecItem dec_item(const DecParams& p, int item, const int* pref) {
    DecItem it;
    it.g = item % p.ngroups;
    const int r = item / p.ngroups;
    if (pref) {   // largest b with pref[b] <= r
        int lo = 0, hi = p.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pref[mid] <= r) lo = mid; else hi = mid - 1;
        }
        it.b = lo;
        it.c = r - pref[lo];
    } else {
        it.b = r % p.B;
        it.c = r / p.B;
    }
    int L = p.cache_len[it.b];
    it.L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
    const long long lo_ll = (long long)it.L - p.W;
    it.lo = lo_ll < 0 ? 0 : int(lo_ll);
    it.start = it.lo + it.c * kDecodeChunk;
    it.end = min(it.start + kDecodeChunk, it.L);
    return it;
}

// Consumer-warp barrier (named barrier 1; warp 0, the producer, never joins it).
__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

template <int D, int QPT, bool kRope>
__global__ void __launch_bounds__(32 + decode_max_consumers(QPT), 1) swa_decode_kernel(const DecParams p) {
    constexpr int LPH = D / 8;                       // threads per (K/V head, query subgroup) pair
    extern __shared__ __align__(128) uint8_t smem[];
    const int H = p.H, kvg = p.kv_group;
    const int ncons = int(blockDim.x) - 32;          // consumer threads (whole warps)
    const uint32_t rowb = uint32_t(p.gh) * D * 2;    // bytes of one slot's K (or V) heads of a group
    const uint32_t stage_bytes = 2u * uint32_t(p.ss) * rowb;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + uint32_t(p.nstage) * stage_bytes;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (p.nstage + s); };
    const uint32_t item_full0 = bar0 + 16u * p.nstage, item_empty0 = item_full0 + 8u * kDecodeItemRing;
    volatile int* misc = reinterpret_cast<volatile int*>(smem + (item_empty0 + 8u * kDecodeItemRing - sbase));
    volatile int* abort_flag = misc;                 // [0] abort, [1] stream slot
    volatile int* ring = misc + 2;                   // kDecodeItemRing entries
    volatile int* is_last = misc + 2 + kDecodeItemRing;
    int* pref = p.B <= kDecodePrefixMax ? const_cast<int*>(misc + 8) : nullptr;   // [B + 1]
    const int tid = threadIdx.x, lane = tid & 31;
    if (pref) {
        // chunks per sequence (chunk 0 always counts), then their exclusive prefix sum: warp 0
        // scans, each lane over a contiguous run of sequences
        for (int b = tid; b < p.B; b += blockDim.x) {
            int L = p.cache_len[b];
            L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
            const long long lo = (long long)L - p.W;
            const int n = L - (lo < 0 ? 0 : int(lo));
            pref[b + 1] = max(1, (n + kDecodeChunk - 1) / kDecodeChunk);
        }
        __syncthreads();
        if (tid < 32) {
            const int per = (p.B + 31) / 32, b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
            int sum = 0;
            for (int b = b0; b < b1; ++b) sum += pref[b + 1];
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            int run = incl - sum;   // chunks of the sequences before b0
            if (tid == 0) pref[0] = 0;
            for (int b = b0; b < b1; ++b) {
                run += pref[b + 1];
                pref[b + 1] = run;
            }
        }
    }

    if (tid == 0) {
        for (int s = 0; s < p.nstage; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), ncons / 32);
        }
        for (int e = 0; e < kDecodeItemRing; ++e) {
            mbar_init(item_full0 + 8u * e, 1);
            mbar_init(item_empty0 + 8u * e, ncons / 32);
        }
        abort_flag[0] = 0;
        abort_flag[1] = p.stream_slot;
        fence_barrier_init();
    }
    __syncthreads();
    const int n_items = pref ? pref[p.B] * p.ngroups : p.n_items;

    if (tid < 32) {
        // ------------------------------ producer: bulk copies of K / V rows ------------------------------
        if (lane == 0) {
            bool ok = true;
            int kq = 0, st = 0;
            for (;; ++kq) {
                int item = 0x7fffffff;
                DecItem g{};
                if (ok && kq >= kDecodeItemRing)
                    ok = mbar_wait(item_empty0 + 8u * (kq % kDecodeItemRing), uint32_t(((kq / kDecodeItemRing) - 1) & 1),
                                   abort_flag, p.wait_limit, kStatusTimeoutProducer);
                while (ok) {   // draw until an item holds window slots (chunk 0 always counts)
                    const int it = atomicAdd(&g_work_slots[p.stream_slot].next, 1);
                    if (it >= n_items) break;
                    g = dec_item(p, it, pref);
                    if (g.start < g.end || g.c == 0) {
                        item = it;
                        break;
                    }
                }
                ring[kq % kDecodeItemRing] = item;
                mbar_arrive(item_full0 + 8u * (kq % kDecodeItemRing));
                if (item == 0x7fffffff) break;
                const int hk0 = g.g * p.gh;
                const int ghe = min(p.gh, p.Hk - hk0);        // heads of this group
                const uint32_t cpy = uint32_t(ghe) * D * 2;
                for (int s0 = g.start; s0 < g.end && ok; s0 += p.ss, ++st) {
                    const int stage = st % p.nstage;
                    if (st >= p.nstage &&
                        !(ok = mbar_wait(empty(stage), uint32_t(((st / p.nstage) - 1) & 1), abort_flag, p.wait_limit,
                                         kStatusTimeoutProducer)))
                        break;
                    const int n = min(p.ss, g.end - s0);
                    const uint32_t dk = sbase + uint32_t(stage) * stage_bytes, dv = dk + uint32_t(p.ss) * rowb;
                    mbar_arrive_expect_tx(full(stage), 2u * uint32_t(n) * cpy);
                    const size_t row0 = (size_t(g.b) * p.cap + size_t(s0)) * p.Hk + hk0;
                    if (ghe == p.Hk) {   // the group is every head: the n slots are one contiguous block
                        bulk_load(dk, p.kc + row0 * D, uint32_t(n) * cpy, full(stage));
                        bulk_load(dv, p.vc + row0 * D, uint32_t(n) * cpy, full(stage));
                    } else {
                        for (int u = 0; u < n; ++u) {
                            bulk_load(dk + uint32_t(u) * rowb, p.kc + (row0 + size_t(u) * p.Hk) * D, cpy, full(stage));
                            bulk_load(dv + uint32_t(u) * rowb, p.vc + (row0 + size_t(u) * p.Hk) * D, cpy, full(stage));
                        }
                    }
                }
            }
            work_slot_finish(p.stream_slot);
            for (int s = 0; s < p.nstage && s < st; ++s)   // no copy may still be landing at exit
                mbar_drain(full(s), uint32_t(((st - s + p.nstage - 1) / p.nstage - 1) & 1), p.wait_limit,
                           p.stream_slot);
        }
        return;
    }

    // ------------------------------ consumers ------------------------------
    const int ct = tid - 32;
    const int lp = ct / LPH;                         // pair within the group
    const int c = ct % LPH;                          // 16-byte piece of the head row
    const unsigned gmask = rope_group_mask<D>();
    bool ok = true;
    int st = 0;
    for (int kq = 0;; ++kq) {
        const int e = kq % kDecodeItemRing;
        ok = ok && __all_sync(0xffffffffu, mbar_wait(item_full0 + 8u * e, uint32_t((kq / kDecodeItemRing) & 1),
                                                     abort_flag, p.wait_limit, kStatusTimeoutSoftmax));
        const int item = ok ? ring[e] : 0x7fffffff;
        __syncwarp();
        if (lane == 0) mbar_arrive(item_empty0 + 8u * e);
        if (item == 0x7fffffff) break;
        const DecItem g = dec_item(p, item, pref);
        const int hk0 = g.g * p.gh;
        const int npairs = min(p.gh, p.Hk - hk0) * p.nsub;
        const bool live = lp < npairs;
        const int pr = live ? lp : 0;
        const int hkl = pr / p.nsub;                 // K/V head within the group (stage row)
        const int hk = hk0 + hkl;
        const int qs = (pr % p.nsub) * QPT;          // first query head of the subgroup within the group
        bool hv[QPT];
        int hq[QPT];
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            hv[a] = live && (qs + a < kvg);
            hq[a] = hk * kvg + min(qs + a, kvg - 1);
        }
        const int L = g.L, b = g.b;
        int rpos = 0;   // position of the new token (kRope)
        if (kRope) {
            rpos = L - 1;
            if (rpos >= p.max_pos) {
                if (ct == 0 && g.c == 0 && g.g == 0) report_status(p.stream_slot, kStatusPositionRange);
                rpos = 0;
            }
            rpos = rpos < 0 ? 0 : rpos;
        }
        float qv[QPT][8];
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            const uint4 u = hv[a] ? *reinterpret_cast<const uint4*>(p.q + (size_t(b) * H + hq[a]) * D + c * 8)
                                  : make_uint4(0, 0, 0, 0);
            bf16x8_to_f32<D>(u, qv[a]);
            if (kRope) {   // every lane of the warp takes part (pairs are whole groups of D/8 lanes)
                rope_qknorm8<D>(qv[a], c, p.rope_cos + size_t(rpos) * (D / 2), p.rope_sin + size_t(rpos) * (D / 2),
                                p.eps, gmask);
                bf16x8_to_f32<D>(bf16x8_pack(qv[a]), qv[a]);   // a bf16 activation, like every other query
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
        for (int s0 = g.start; s0 < g.end && ok; s0 += p.ss, ++st) {
            const int stage = st % p.nstage;
            ok = __all_sync(0xffffffffu, mbar_wait(full(stage), uint32_t((st / p.nstage) & 1), abort_flag,
                                                   p.wait_limit, kStatusTimeoutSoftmax));
            if (!ok) break;
            const int n = min(p.ss, g.end - s0);
            uint8_t* sk = smem + size_t(stage) * stage_bytes + size_t(hkl) * D * 2 + c * 16;
            uint8_t* sv = sk + size_t(p.ss) * rowb;
            if (kRope && L - 1 >= s0 && L - 1 < s0 + n && L - 1 < p.max_pos) {
                // The new token's slot is in this stage: its rotated, normalised key and its value go
                // into the cache, and into the staged copy that this thread (the only reader of its
                // piece, with the other subgroups of its K/V head, which write the same bytes) reads.
                const size_t src = (size_t(b) * p.Hk + hk) * D + c * 8;
                float f[8];
                bf16x8_to_f32<D>(*reinterpret_cast<const uint4*>(p.k_new + src), f);
                rope_qknorm8<D>(f, c, p.rope_cos + size_t(rpos) * (D / 2), p.rope_sin + size_t(rpos) * (D / 2), p.eps,
                                gmask);
                const uint4 kw = bf16x8_pack(f), vw = *reinterpret_cast<const uint4*>(p.v_new + src);
                if (live) {
                    const size_t dst = (size_t(b) * p.cap + size_t(L - 1)) * (size_t(p.Hk) * D) + size_t(hk) * D + c * 8;
                    *reinterpret_cast<uint4*>(p.kc_out + dst) = kw;
                    *reinterpret_cast<uint4*>(p.vc_out + dst) = vw;
                    *reinterpret_cast<uint4*>(sk + size_t(L - 1 - s0) * rowb) = kw;
                    *reinterpret_cast<uint4*>(sv + size_t(L - 1 - s0) * rowb) = vw;
                }
            }
            for (int u0 = 0; u0 < n; u0 += kDecodeUnroll) {
                uint4 ku[kDecodeUnroll], vu[kDecodeUnroll];
#pragma unroll
                for (int u = 0; u < kDecodeUnroll; ++u) {
                    const bool in = u0 + u < n;
                    ku[u] = in ? *reinterpret_cast<const uint4*>(sk + size_t(u0 + u) * rowb) : make_uint4(0, 0, 0, 0);
                    vu[u] = in ? *reinterpret_cast<const uint4*>(sv + size_t(u0 + u) * rowb) : make_uint4(0, 0, 0, 0);
                }
                float sc[QPT][kDecodeUnroll];
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
                    for (int a = 0; a < QPT; ++a) sc[a][u] = (u0 + u < n) ? d[a] : -INFINITY;
                }
#pragma unroll
                for (int a = 0; a < QPT; ++a) {
                    float mx = m[a];
#pragma unroll
                    for (int u = 0; u < kDecodeUnroll; ++u) mx = fmaxf(mx, sc[a][u]);
                    const float alpha = ex2_approx(m[a] - mx);   // m = -inf on the first batch: alpha = 0
                    l[a] *= alpha;
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[a][i] *= alpha;
                    m[a] = mx;
                }
#pragma unroll
                for (int u = 0; u < kDecodeUnroll; ++u) {
                    float vf[8];
                    bf16x8_to_f32<D>(vu[u], vf);
#pragma unroll
                    for (int a = 0; a < QPT; ++a) {
                        const float pu = ex2_approx(sc[a][u] - m[a]);   // 0 for padding (-inf)
                        l[a] += pu;
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[a][i] = fmaf(pu, vf[i], acc[a][i]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(stage));   // this warp has read the stage
        }
        if (!ok) break;

        // ---- partials of this chunk ----
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            if (!hv[a]) continue;
            const size_t pidx = (size_t(b) * p.nsplit_max + g.c) * H + hq[a];
            float4* po = reinterpret_cast<float4*>(p.part_o + pidx * D + c * 8);
            po[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            po[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
            if (c == 0) {
                p.part_ml[2 * pidx] = m[a];
                p.part_ml[2 * pidx + 1] = l[a];
            }
        }
        const int nwin = L - g.lo;
        const int used = max(1, (nwin + kDecodeChunk - 1) / kDecodeChunk);   // chunks of this sequence
        int* ticket = p.tickets + size_t(b) * p.ngroups + g.g;
        __threadfence();
        consumer_sync(ncons);
        if (ct == 0) *is_last = (atomicAdd(ticket, 1) == used - 1);
        consumer_sync(ncons);
        if (!*is_last) continue;
        __threadfence();

        // ---- last chunk of this (sequence, head group): merge the partials in one pass with a
        // running maximum; the loads of MB partials of every query head of the thread are in flight
        // together.  Every used chunk but an empty chunk 0 holds at least one slot. ----
        constexpr int MB = QPT >= 3 ? 2 : 4;
        float M[QPT], lsum[QPT], o8[QPT][8];
#pragma unroll
        for (int a = 0; a < QPT; ++a) {
            M[a] = -INFINITY;
            lsum[a] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[a][i] = 0.f;
        }
        const size_t pbase = size_t(b) * p.nsplit_max * H;   // partial (chunk sp, head h) at pbase + sp * H + h
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
                    oa[a][u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8))
                                  : make_float4(0, 0, 0, 0);
                    ob[a][u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8) + 1)
                                  : make_float4(0, 0, 0, 0);
                }
#pragma unroll
            for (int a = 0; a < QPT; ++a) {
                float bm = M[a];
#pragma unroll
                for (int u = 0; u < MB; ++u) bm = fmaxf(bm, ml[a][u][0]);
                if (bm == -INFINITY) continue;                 // nothing yet (or an empty window)
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
            const bool any = M[a] != -INFINITY;
            const float inv = any ? 1.f / lsum[a] : 0.f;
            uint4 w;
            w.x = pack_bf16x2(o8[a][0] * inv, o8[a][1] * inv);
            w.y = pack_bf16x2(o8[a][2] * inv, o8[a][3] * inv);
            w.z = pack_bf16x2(o8[a][4] * inv, o8[a][5] * inv);
            w.w = pack_bf16x2(o8[a][6] * inv, o8[a][7] * inv);
            *reinterpret_cast<uint4*>(p.o + (size_t(b) * H + hq[a]) * D + c * 8) = w;
            if (c == 0 && p.lse != nullptr)
                p.lse[size_t(b) * H + hq[a]] = any ? (M[a] + log2f(lsum[a])) * 0.69314718055994530942f : -INFINITY;
        }
        if (ct == 0) *ticket = 0;   // ready for the next call
    }
}

}  // namespace swa
