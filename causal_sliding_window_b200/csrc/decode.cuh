// decode.cuh -- single-token decode over a KV cache, split along the cache.
//
// The inference engine keeps a per-layer K/V cache and attends the new token
// to it through flash_attn_with_kvcache (apidog guide "Train your own
// ChatGPT", section 6 "Inference engine", KV cache).  Sequence b holds
// L = cache_len[b] tokens; the new query sits at position L-1 and attends to
// slots max(0, L-W) .. L-1 of its cache.
//
// Layout: caches [B, cap, H, D] bf16, so one cache slot of one sequence is a
// contiguous H*D*2-byte row (3 KB at H=12, D=128).  A CTA takes a chunk of
// CHUNK consecutive slots of one sequence and a group of up to kDecodeThreads*8/D consecutive
// heads (4 at D = 128): thread slot (h, c) owns the 16-byte piece c of head h, so each slot's
// heads of the group are read as one contiguous, coalesced, vectorised sweep (1 KB at D = 128).
// Small head groups put more CTAs, and so more loads, in flight (measured: 64 threads per CTA
// beat 256 by about 4% on the decode workload).  Per head, the D/8 threads reduce q.k
// with warp shuffles and keep an online softmax (m, l) and 8 output
// accumulators in registers.  Each CTA writes its partial (m, l, o) to the
// workspace; the last CTA of a sequence (atomic ticket) merges the partials:
//   M = max_c m_c,  l = sum_c 2^(m_c - M) l_c,  o = sum_c 2^(m_c - M) o_c / l.
// Slots outside the window are never read.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace swa {

constexpr int kDecodeChunk = 128;  // cache slots per CTA
constexpr int kDecodeUnroll = 4;   // slots per batch (two batches in flight per thread)

struct DecParams {
    const __nv_bfloat16* q;        // [B,H,D]
    const __nv_bfloat16* kc;       // [B,cap,Hk,D], Hk = H / kv_group
    const __nv_bfloat16* vc;
    const int32_t* cache_len;      // [B]
    __nv_bfloat16* o;              // [B,H,D]
    float* lse;                    // [B,H] or null
    int* counters;                 // [B, n_hgroup], zero between calls
    float* part_ml;                // [B, nsplit_max, H, 2]
    float* part_o;                 // [B, nsplit_max, H, D]
    int B, cap, H;
    int kv_group;                  // query heads per K/V head: query head h reads cache head h / kv_group
    long long W;
    float scale_log2;
    int nsplit;                    // splits launched per sequence
    int nsplit_max;                // stride of the partial arrays
};

constexpr int kDecodeThreads = 64;   // threads per CTA: D/8 per head, so 4 heads of D = 128 (more CTAs in flight)

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

template <int D>
__global__ void __launch_bounds__(kDecodeThreads) swa_decode_kernel(const DecParams p) {
    constexpr int LPH = D / 8;                       // threads per head
    constexpr int G = kDecodeThreads / LPH;          // heads per CTA
    const int split = blockIdx.x, b = blockIdx.y, hg = blockIdx.z;
    const int H = p.H;
    const int h0 = hg * G;
    const int slots = min(G, H - h0) * LPH;
    const int tid = threadIdx.x;
    const bool live = tid < slots;
    const int h = h0 + (live ? tid / LPH : 0);
    const int c = tid % LPH;
    int* counter = p.counters + size_t(b) * gridDim.z + hg;

    int L = p.cache_len[b];
    L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
    const long long lo_ll = (long long)L - p.W;
    const int lo = lo_ll < 0 ? 0 : int(lo_ll);
    const int start = lo + split * kDecodeChunk;
    const int end = min(start + kDecodeChunk, L);

    float qv[8];
    {
        const uint4 u = live ? *reinterpret_cast<const uint4*>(p.q + (size_t(b) * H + h) * D + c * 8) : make_uint4(0, 0, 0, 0);
        bf16x8_to_f32<D>(u, qv);
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[i] *= p.scale_log2;
    }
    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    const size_t row_elems = size_t(H / p.kv_group) * D;   // one cache slot: all K/V heads
    const int hk = h / p.kv_group;
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
        float s[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            float kf[8];
            bf16x8_to_f32<D>(ku[u], kf);
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) d = fmaf(qv[i], kf[i], d);
#pragma unroll
            for (int off = LPH / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            s[u] = (pos + u < end) ? d : -INFINITY;
        }
        float mx = m;
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) mx = fmaxf(mx, s[u]);
        const float alpha = ex2_approx(m - mx);   // m = -inf on the first batch: alpha = 0
        l *= alpha;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const float pu = ex2_approx(s[u] - mx);
            l += pu;
            float vf[8];
            bf16x8_to_f32<D>(vu[u], vf);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(pu, vf[i], acc[i]);
        }
        m = mx;
    };
    uint4 ka[kDecodeUnroll], va[kDecodeUnroll], kn[kDecodeUnroll], vn[kDecodeUnroll];
    if (start < end) load(start, ka, va);
    for (int pos = start; pos < end; pos += 2 * kDecodeUnroll) {   // CTA-uniform trip count
        if (pos + kDecodeUnroll < end) load(pos + kDecodeUnroll, kn, vn);
        consume(pos, ka, va);
        if (pos + 2 * kDecodeUnroll < end) load(pos + 2 * kDecodeUnroll, ka, va);
        if (pos + kDecodeUnroll < end) consume(pos + kDecodeUnroll, kn, vn);
    }

    // ---- partial of this chunk ----
    const size_t pidx = (size_t(b) * p.nsplit_max + split) * H + h;
    if (live) {
        float4* po = reinterpret_cast<float4*>(p.part_o + pidx * D + c * 8);
        po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (c == 0) {
            p.part_ml[2 * pidx] = m;
            p.part_ml[2 * pidx + 1] = l;
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

    // ---- last CTA of this sequence: merge the partials of the non-empty chunks ----
    const int n = L - lo;
    const int used = (n + kDecodeChunk - 1) / kDecodeChunk;
    if (live) {
        // Partials are read in batches so their load latencies overlap.
        const size_t pbase = (size_t(b) * p.nsplit_max) * H + h;   // partial (split sp) at pbase + sp * H
        float M = -INFINITY;
        for (int sp0 = 0; sp0 < used; sp0 += 8) {
            float mv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                mv[u] = (sp0 + u < used) ? __ldcg(p.part_ml + 2 * (pbase + size_t(sp0 + u) * H)) : -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) M = fmaxf(M, mv[u]);
        }
        float lsum = 0.f, o8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o8[i] = 0.f;
        for (int sp0 = 0; sp0 < used; sp0 += 4) {
            float ml[4][2];
            float4 oa[4], ob[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const bool in = sp0 + u < used;
                const size_t q = pbase + size_t(sp0 + u) * H;
                ml[u][0] = in ? __ldcg(p.part_ml + 2 * q) : -INFINITY;
                ml[u][1] = in ? __ldcg(p.part_ml + 2 * q + 1) : 0.f;
                oa[u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8)) : make_float4(0, 0, 0, 0);
                ob[u] = in ? __ldcg(reinterpret_cast<const float4*>(p.part_o + q * D + c * 8) + 1)
                           : make_float4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float w = ex2_approx(ml[u][0] - M);   // 0 for empty partials (m = -inf)
                lsum = fmaf(w, ml[u][1], lsum);
                o8[0] = fmaf(w, oa[u].x, o8[0]);
                o8[1] = fmaf(w, oa[u].y, o8[1]);
                o8[2] = fmaf(w, oa[u].z, o8[2]);
                o8[3] = fmaf(w, oa[u].w, o8[3]);
                o8[4] = fmaf(w, ob[u].x, o8[4]);
                o8[5] = fmaf(w, ob[u].y, o8[5]);
                o8[6] = fmaf(w, ob[u].z, o8[6]);
                o8[7] = fmaf(w, ob[u].w, o8[7]);
            }
        }
        const float inv = used > 0 ? 1.f / lsum : 0.f;
        uint4 w;
        w.x = pack_bf16x2(o8[0] * inv, o8[1] * inv);
        w.y = pack_bf16x2(o8[2] * inv, o8[3] * inv);
        w.z = pack_bf16x2(o8[4] * inv, o8[5] * inv);
        w.w = pack_bf16x2(o8[6] * inv, o8[7] * inv);
        *reinterpret_cast<uint4*>(p.o + (size_t(b) * H + h) * D + c * 8) = w;
        if (c == 0 && p.lse != nullptr)
            p.lse[size_t(b) * H + h] = used > 0 ? (M + log2f(lsum)) * 0.69314718055994530942f : -INFINITY;
    }
    if (tid == 0) *counter = 0;   // ready for the next call
}

}  // namespace swa
