// rope.cuh -- rotary embedding + QK norm, the prologue of attention in the GPT model
// (apidog guide "Train your own ChatGPT", section 1 "GPT model", architecture features: rotary
// embeddings and QK normalisation, an RMSNorm without learnable parameters).
//
// For one head vector x in R^D at position pos (pairs (x[i], x[i + D/2]), i < D/2):
//   r1 = x1 cos(pos th_i) - x2 sin(pos th_i),  r2 = x1 sin(pos th_i) + x2 cos(pos th_i),
//   y  = r / sqrt(mean(r^2) + eps),            th_i = base^(-2i/D)   (RoFormer rotation).
// cos / sin come from tables [max_pos, D/2] fp32 that the caller owns (swa_rope_tables_kernel
// fills them for a given base).  The rotation keeps |x|, so it commutes with the norm.
//
// Layout: a row (one head vector) is D/8 consecutive threads of a warp, each holding 8
// consecutive elements (16 bytes); the partner of piece c is piece c ^ (D/16) (the same
// offset in the other half), fetched with a shuffle, and mean(r^2) is a shuffle reduction
// over the row's threads.  Rows never straddle a warp (D/8 divides 32).
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace swa {

// Lanes of the row group of this thread (D/8 consecutive lanes).
template <int D>
__device__ __forceinline__ unsigned rope_group_mask() {
    constexpr int CPR = D / 8;
    constexpr unsigned ones = CPR == 32 ? 0xffffffffu : ((1u << CPR) - 1u);
    return ones << ((threadIdx.x & 31) & ~(CPR - 1));
}

// Rotation of this thread's 8 elements (piece c of a row) at the position whose table rows are
// cs / sn, in place: on return x holds r.  All threads of the row group call it together.
template <int D>
__device__ __forceinline__ void rope_rotate8(float (&x)[8], int c, const float* cs, const float* sn,
                                             unsigned mask, bool inverse) {
    constexpr int HALF = D / 16;   // pieces per half row
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = __shfl_xor_sync(mask, x[i], HALF);
    const bool first = c < HALF;
    const int i0 = (first ? c : c - HALF) * 8;
    const float4 c0 = *reinterpret_cast<const float4*>(cs + i0), c1 = *reinterpret_cast<const float4*>(cs + i0 + 4);
    const float4 s0 = *reinterpret_cast<const float4*>(sn + i0), s1 = *reinterpret_cast<const float4*>(sn + i0 + 4);
    const float co[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    float si[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    if (inverse) {
#pragma unroll
        for (int i = 0; i < 8; ++i) si[i] = -si[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)   // first half: x1 c - x2 s (partner = x2); second: x1 s + x2 c (partner = x1)
        x[i] = first ? fmaf(x[i], co[i], -p[i] * si[i]) : fmaf(p[i], si[i], x[i] * co[i]);
}

// Sum over the row group.
template <int D>
__device__ __forceinline__ float rope_row_sum(float v, unsigned mask) {
#pragma unroll
    for (int off = D / 16; off > 0; off >>= 1) v += __shfl_xor_sync(mask, v, off);
    return v;
}

// y = rope(x) / sqrt(mean(rope(x)^2) + eps) for this thread's piece, in place.
template <int D>
__device__ __forceinline__ void rope_qknorm8(float (&x)[8], int c, const float* cs, const float* sn, float eps,
                                             unsigned mask) {
    rope_rotate8<D>(x, c, cs, sn, mask, false);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
    const float ms = rope_row_sum<D>(ss, mask) * (1.f / D) + eps;
    const float inv = ms > 0.f ? rsqrtf(ms) : 0.f;   // an all-zero row with eps = 0 stays zero
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] *= inv;
}

__device__ __forceinline__ void bf16x8_unpack(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h2[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ uint4 bf16x8_pack(const float (&f)[8]) {
    uint4 w;
    w.x = pack_bf16x2(f[0], f[1]);
    w.y = pack_bf16x2(f[2], f[3]);
    w.z = pack_bf16x2(f[4], f[5]);
    w.w = pack_bf16x2(f[6], f[7]);
    return w;
}

// cos / sin tables [max_pos, half] for th_i = base^(-2i/D), D = 2 * half; angles in double so that
// positions in the hundreds of thousands keep full fp32 accuracy.
__global__ void __launch_bounds__(256) swa_rope_tables_kernel(float* __restrict__ cs, float* __restrict__ sn,
                                                              int max_pos, int half, double base) {
    const long long total = (long long)max_pos * half;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int i = int(e % half);
        const long long pos = e / half;
        const double ang = double(pos) * pow(base, -double(i) / double(half));
        cs[e] = float(cos(ang));
        sn[e] = float(sin(ang));
    }
}

// Position of token t of sequence b, or -1 (status flagged) when it has no table row.
__device__ __forceinline__ int rope_position(const int* pos0, int b, int t, int max_pos, int slot) {
    const long long pos = (long long)(pos0 ? pos0[b] : 0) + t;
    if (pos < 0 || pos >= max_pos) {
        report_status(slot, kStatusPositionRange);
        return -1;
    }
    return int(pos);
}

// Forward: y[b,t,h,:] = rope+norm of x[b,t,h,:] at position pos0[b] + t (pos0 NULL: t).
// kBwd: dx from dy instead, with r = rope(x), s = (mean(r^2) + eps)^(-1/2):
//   dr = s dy - (s^3 / D) r (dy . r),  dx = rope^(-1)(dr).
// A row whose position has no table row is left unwritten.
// x, dy and y may be the same array (in place): no __restrict__ on them.  Each thread reads its own
// 16 bytes before writing them, and partner values travel through shuffles, not memory.
template <int D, bool kBwd>
__global__ void __launch_bounds__(256) swa_rope_qknorm_kernel(const __nv_bfloat16* x, const __nv_bfloat16* dy,
                                                              __nv_bfloat16* y, int B, int T, int H,
                                                              const int* __restrict__ pos0,
                                                              const float* __restrict__ cs,
                                                              const float* __restrict__ sn, int max_pos, float eps,
                                                              int slot) {
    constexpr int CPR = D / 8;
    const long long total = (long long)B * T * H * CPR;   // a multiple of CPR: rows are whole
    const unsigned mask = rope_group_mask<D>();
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int c = int(e % CPR);
        const long long row = e / CPR;   // (b, t, h)
        const int t = int((row / H) % T);
        const int b = int(row / ((long long)H * T));
        const int pos = rope_position(pos0, b, t, max_pos, slot);
        if (pos < 0) continue;   // uniform over the row group
        const float* crow = cs + (size_t)pos * (D / 2);
        const float* srow = sn + (size_t)pos * (D / 2);
        float v[8];
        bf16x8_unpack(*reinterpret_cast<const uint4*>(x + e * 8), v);
        if (!kBwd) {
            rope_qknorm8<D>(v, c, crow, srow, eps, mask);
        } else {
            float g[8];
            bf16x8_unpack(*reinterpret_cast<const uint4*>(dy + e * 8), g);
            rope_rotate8<D>(v, c, crow, srow, mask, false);   // v = r
            float ss = 0.f, gr = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ss = fmaf(v[i], v[i], ss);
                gr = fmaf(g[i], v[i], gr);
            }
            ss = rope_row_sum<D>(ss, mask);
            gr = rope_row_sum<D>(gr, mask);
            const float s = rsqrtf(ss * (1.f / D) + eps);
            const float k3 = s * s * s * (1.f / D) * gr;
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = fmaf(s, g[i], -k3 * v[i]);   // dr
            rope_rotate8<D>(v, c, crow, srow, mask, true);                  // dx = rope^-1(dr)
        }
        *reinterpret_cast<uint4*>(y + e * 8) = bf16x8_pack(v);
    }
}

}  // namespace swa
