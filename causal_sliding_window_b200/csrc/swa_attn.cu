// swa_attn.cu -- C-ABI entry points of libswa_b200.so (declared in include/swa_attn.h).
//
// Host side only: argument validation, TMA tensor maps, workspace carving and
// kernel launches on the caller's stream.  No allocation, no synchronisation
// (except attn_device_status, which is documented to synchronise).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/swa_attn.h"
#include "bwd.cuh"
#include "decode.cuh"
#include "fwd.cuh"
#include "rope.cuh"

namespace {

using namespace swa;

constexpr long long kDefaultWaitLimit = 1LL << 33;   // ~4 s of SM clocks

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [B, T, H, D] bf16 viewed as a 4-D tensor (D, H, T, B), boxes of 64 x 1 x 128 x 1
// with 128-byte swizzle (one box = 128 rows of one head, 64 columns).
bool make_bthd_map(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T), cuuint64_t(B)};
    cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2, cuuint64_t(T) * H * D * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// cudaFuncSetAttribute for the large-shared-memory kernels, once per (device, kernel).
bool ensure_smem(const void* func, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void*>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> g(mu);
    if (done.count({dev, func})) return true;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done.insert({dev, func});
    return true;
}

// Work-counter slot for the next persistent launch (round robin over kWorkSlots, so that
// up to kWorkSlots launches may be in flight at once on different streams).
int next_work_slot() {
    static std::atomic<unsigned> ctr{0};
    return int(ctr.fetch_add(1, std::memory_order_relaxed) % unsigned(kWorkSlots));
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && cache[dev] > 0) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cache[dev] = n;
    return n;
}

bool valid_common(int B, int T, int H, int D, int W, float scale) {
    if (B < 1 || T < 1 || H < 1 || W < 1) return false;
    if (!(scale > 0.f) || scale != scale || scale > 3.4e38f) return false;
    (void)D;
    return true;
}

// Grouped K/V heads: Hkv >= 1 and divides H.
bool valid_kv_heads(int H, int Hkv) { return Hkv >= 1 && H >= 1 && H % Hkv == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Optional events recorded between the three launches of attn_bwd (see
// attn_bwd_set_profile_events); per calling thread.
thread_local cudaEvent_t g_ev_after_pre = nullptr;
thread_local cudaEvent_t g_ev_after_main = nullptr;

int launch_status() { return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH; }

int grid_for(long long work_items, int threads) {
    long long blocks = (work_items + threads - 1) / threads;
    const long long cap = 148LL * 32;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return int(blocks);
}

__global__ void swa_selftest_wait_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t a = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(a, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Nobody arrives on this barrier: the wait must give up after limit_cycles.
    if (threadIdx.x == 0) mbar_wait(a, 0, &abort_flag, limit_cycles, kStatusTimeoutSelftest);
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Fixed decode scratch for callers that cannot allocate device memory
// (attn_decode_noalloc).  Every GPU that loads this library holds the array
// until the process exits.  Host code may not pass the array's name to a
// kernel (on the host it is only a stand-in symbol); its device address is
// looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device (set up on first use per device).
void* noalloc_scratch() {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    if (addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

int attn_fwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B,
                 int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, T, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    const int n_qblk = (T + 255) / 256;
    const long long n_items = (long long)n_qblk * B * H;
    if (n_items > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    const long long grid = n_items < sm_count() ? n_items : sm_count();   // persistent: one CTA per SM
    CUtensorMap mq, mk, mv;
    if (!make_bthd_map(&mq, q, B, T, H, D) || !make_bthd_map(&mk, k, B, T, Hkv, D) ||
        !make_bthd_map(&mv, v, B, T, Hkv, D))
        return ATTN_ERR_LAUNCH;
    FwdParams p;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.T = T;
    p.H = H;
    p.G = H / Hkv;
    p.q_offset = nullptr;
    p.W = W;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_qblk = n_qblk;
    p.n_items = int(n_items);
    p.work_slot = next_work_slot();
    p.wait_limit = kDefaultWaitLimit;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (D == 128) {
        if (!ensure_smem((const void*)swa_fwd_kernel<128>, FwdCfg<128>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_fwd_kernel<128><<<unsigned(grid), FwdCfg<128>::THREADS, FwdCfg<128>::SMEM, s>>>(mq, mk, mv, p);
    } else {
        if (!ensure_smem((const void*)swa_fwd_kernel<64>, FwdCfg<64>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_fwd_kernel<64><<<unsigned(grid), FwdCfg<64>::THREADS, FwdCfg<64>::SMEM, s>>>(mq, mk, mv, p);
    }
    return launch_status();
}

int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B, int T,
             int H, int D, int W, float scale, void* stream) {
    return attn_fwd_gqa(q, k, v, o, lse, B, T, H, H, D, W, scale, stream);
}

// RoPE arguments shared by the fused entry points (null table pointers: no rotation).
struct RopeArgs {
    const float* cs = nullptr;
    const float* sn = nullptr;
    int max_pos = 0;
    float eps = 0.f;
};

static bool valid_rope(const float* cs, const float* sn, int max_pos, float eps) {
    return cs && sn && aligned16(cs) && aligned16(sn) && max_pos >= 1 && eps >= 0.f && std::isfinite(eps);
}

// Launches the append kernel: k_new / v_new rows to slots cache_len[b] + len_off + t, tail zeroed
// up to the 128-slot tile end when tail > 0; keys rotated and normalised when rope.cs is set.
static int launch_append(const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache, attn_bf16* v_cache,
                         const int32_t* cache_len, int B, int Tn, int cap, int Hkv, int D, int len_off, int tail,
                         const RopeArgs& rope, cudaStream_t s) {
    const long long chunks = (long long)B * (Tn + tail) * Hkv * (D / 8);
    const long long blocks = std::min<long long>((chunks + 255) / 256, 148LL * 16);
    const auto* kn = reinterpret_cast<const __nv_bfloat16*>(k_new);
    const auto* vn = reinterpret_cast<const __nv_bfloat16*>(v_new);
    auto* kc = reinterpret_cast<__nv_bfloat16*>(k_cache);
    auto* vc = reinterpret_cast<__nv_bfloat16*>(v_cache);
    const bool r = rope.cs != nullptr;
#define SWA_APPEND(DD, RR)                                                                                    \
    swa_append_kernel<DD, RR><<<unsigned(blocks), 256, 0, s>>>(kn, vn, kc, vc, cache_len, B, Tn, cap, Hkv, len_off, \
                                                               tail, rope.cs, rope.sn, rope.max_pos, rope.eps)
    if (D == 128) {
        if (r) SWA_APPEND(128, true); else SWA_APPEND(128, false);
    } else {
        if (r) SWA_APPEND(64, true); else SWA_APPEND(64, false);
    }
#undef SWA_APPEND
    return launch_status();
}

static int prefill_impl(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                        attn_bf16* v_cache, const int32_t* cache_len, attn_bf16* o, float* lse, int B, int Tn,
                        int cap, int H, int Hkv, int D, int W, float scale, const RopeArgs& rope,
                        attn_bf16* q_rot, void* stream) {
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_len || !o || !lse) return ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k_new, v_new, k_cache, v_cache, o, lse};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cache_len) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, Tn, H, D, W, scale) || !valid_kv_heads(H, Hkv) || cap < Tn) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    const int n_qblk = (Tn + 255) / 256;
    const long long n_items = (long long)n_qblk * B * H;
    if (n_items > 0x7fffffffLL || (long long)B * (Tn + 128) * Hkv * (D / 8) > (1LL << 40)) return ATTN_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // 0. with RoPE: the chunk's queries rotated and normalised at positions cache_len[b] + t
    const attn_bf16* q_in = q;
    if (rope.cs) {
        const long long rows = (long long)B * Tn * H * (D / 8);
        const unsigned blocks = unsigned(std::min<long long>((rows + 255) / 256, 148LL * 16));
        const auto* x = reinterpret_cast<const __nv_bfloat16*>(q);
        auto* y = reinterpret_cast<__nv_bfloat16*>(q_rot);
        if (D == 128)
            swa_rope_qknorm_kernel<128, false><<<blocks, 256, 0, s>>>(x, nullptr, y, B, Tn, H, cache_len, rope.cs,
                                                                       rope.sn, rope.max_pos, rope.eps);
        else
            swa_rope_qknorm_kernel<64, false><<<blocks, 256, 0, s>>>(x, nullptr, y, B, Tn, H, cache_len, rope.cs,
                                                                      rope.sn, rope.max_pos, rope.eps);
        if (launch_status() != ATTN_OK) return ATTN_ERR_LAUNCH;
        q_in = q_rot;
    }
    // 1. append the chunk's K / V (and zero the rest of its last 128-slot tile)
    if (launch_append(k_new, v_new, k_cache, v_cache, cache_len, B, Tn, cap, Hkv, D, 0, 128, rope, s) != ATTN_OK)
        return ATTN_ERR_LAUNCH;
    // 2. the forward of the chunk's queries at absolute positions cache_len[b] + t over the cache
    const long long grid = n_items < sm_count() ? n_items : sm_count();
    CUtensorMap mq, mk, mv;
    if (!make_bthd_map(&mq, q_in, B, Tn, H, D) || !make_bthd_map(&mk, k_cache, B, cap, Hkv, D) ||
        !make_bthd_map(&mv, v_cache, B, cap, Hkv, D))
        return ATTN_ERR_LAUNCH;
    FwdParams p;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.T = Tn;
    p.H = H;
    p.G = H / Hkv;
    p.q_offset = cache_len;
    p.W = W;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_qblk = n_qblk;
    p.n_items = int(n_items);
    p.work_slot = next_work_slot();
    p.wait_limit = kDefaultWaitLimit;
    if (D == 128) {
        if (!ensure_smem((const void*)swa_fwd_kernel<128, true>, FwdCfg<128>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_fwd_kernel<128, true><<<unsigned(grid), FwdCfg<128>::THREADS, FwdCfg<128>::SMEM, s>>>(mq, mk, mv, p);
    } else {
        if (!ensure_smem((const void*)swa_fwd_kernel<64, true>, FwdCfg<64>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_fwd_kernel<64, true><<<unsigned(grid), FwdCfg<64>::THREADS, FwdCfg<64>::SMEM, s>>>(mq, mk, mv, p);
    }
    return launch_status();
}

int attn_prefill(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                 attn_bf16* v_cache, const int32_t* cache_len, attn_bf16* o, float* lse, int B, int Tn, int cap,
                 int H, int Hkv, int D, int W, float scale, void* stream) {
    return prefill_impl(q, k_new, v_new, k_cache, v_cache, cache_len, o, lse, B, Tn, cap, H, Hkv, D, W, scale,
                        RopeArgs{}, nullptr, stream);
}

size_t attn_prefill_rope_workspace_bytes(int B, int Tn, int H, int D) {
    if (B < 1 || Tn < 1 || H < 1 || (D != 64 && D != 128)) return 0;
    return align256(size_t(B) * Tn * H * D * 2);
}

int attn_prefill_rope(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                      attn_bf16* v_cache, const int32_t* cache_len, const float* rope_cos, const float* rope_sin,
                      int max_pos, float eps, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                      int Tn, int cap, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!valid_rope(rope_cos, rope_sin, max_pos, eps) || !workspace) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_prefill_rope_workspace_bytes(B, Tn, H, D);
    if (need != 0 && ws_bytes < need) return ATTN_ERR_WORKSPACE;
    RopeArgs r;
    r.cs = rope_cos;
    r.sn = rope_sin;
    r.max_pos = max_pos;
    r.eps = eps;
    return prefill_impl(q, k_new, v_new, k_cache, v_cache, cache_len, o, lse, B, Tn, cap, H, Hkv, D, W, scale, r,
                        static_cast<attn_bf16*>(workspace), stream);
}

int attn_rope_tables(float* rope_cos, float* rope_sin, int max_pos, int D, double base, void* stream) {
    if (!rope_cos || !rope_sin || !aligned16(rope_cos) || !aligned16(rope_sin)) return ATTN_ERR_INVALID_ARG;
    if (max_pos < 1 || D < 2 || D % 2 != 0 || !(base > 1.0) || !std::isfinite(base)) return ATTN_ERR_INVALID_ARG;
    const long long total = (long long)max_pos * (D / 2);
    const unsigned blocks = unsigned(std::min<long long>((total + 255) / 256, 148LL * 16));
    swa_rope_tables_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(rope_cos, rope_sin, max_pos,
                                                                                       D / 2, base);
    return launch_status();
}

static int rope_qknorm_impl(const attn_bf16* x, const attn_bf16* dy, attn_bf16* y, const int32_t* pos0,
                            const float* rope_cos, const float* rope_sin, int max_pos, int B, int T, int H, int D,
                            float eps, bool bwd, void* stream) {
    if (!x || !y || (bwd && !dy) || !aligned16(x) || !aligned16(y) || (bwd && !aligned16(dy)))
        return ATTN_ERR_INVALID_ARG;
    if (pos0 && (reinterpret_cast<uintptr_t>(pos0) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_rope(rope_cos, rope_sin, max_pos, eps) || B < 1 || T < 1 || H < 1) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    const long long rows = (long long)B * T * H * (D / 8);
    const unsigned blocks = unsigned(std::min<long long>((rows + 255) / 256, 148LL * 16));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const auto* xx = reinterpret_cast<const __nv_bfloat16*>(x);
    const auto* gg = reinterpret_cast<const __nv_bfloat16*>(dy);
    auto* yy = reinterpret_cast<__nv_bfloat16*>(y);
#define SWA_ROPE(DD, BB) \
    swa_rope_qknorm_kernel<DD, BB><<<blocks, 256, 0, s>>>(xx, gg, yy, B, T, H, pos0, rope_cos, rope_sin, max_pos, eps)
    if (D == 128) {
        if (bwd) SWA_ROPE(128, true); else SWA_ROPE(128, false);
    } else {
        if (bwd) SWA_ROPE(64, true); else SWA_ROPE(64, false);
    }
#undef SWA_ROPE
    return launch_status();
}

int attn_rope_qknorm(const attn_bf16* x, attn_bf16* y, const int32_t* pos0, const float* rope_cos,
                     const float* rope_sin, int max_pos, int B, int T, int H, int D, float eps, void* stream) {
    return rope_qknorm_impl(x, nullptr, y, pos0, rope_cos, rope_sin, max_pos, B, T, H, D, eps, false, stream);
}

int attn_rope_qknorm_bwd(const attn_bf16* x, const attn_bf16* dy, attn_bf16* dx, const int32_t* pos0,
                         const float* rope_cos, const float* rope_sin, int max_pos, int B, int T, int H, int D,
                         float eps, void* stream) {
    return rope_qknorm_impl(x, dy, dx, pos0, rope_cos, rope_sin, max_pos, B, T, H, D, eps, true, stream);
}

int attn_fwd_rope(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* q_rot, attn_bf16* k_rot,
                  attn_bf16* o, float* lse, const float* rope_cos, const float* rope_sin, int max_pos, float eps,
                  int B, int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!q || !k || !v || !q_rot || !k_rot || !o || !lse) return ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, q_rot, k_rot, o, lse};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, T, H, D, W, scale) || !valid_kv_heads(H, Hkv) || !valid_rope(rope_cos, rope_sin, max_pos, eps))
        return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    int st = rope_qknorm_impl(q, nullptr, q_rot, nullptr, rope_cos, rope_sin, max_pos, B, T, H, D, eps, false, stream);
    if (st == ATTN_OK)
        st = rope_qknorm_impl(k, nullptr, k_rot, nullptr, rope_cos, rope_sin, max_pos, B, T, Hkv, D, eps, false, stream);
    if (st == ATTN_OK) st = attn_fwd_gqa(q_rot, k_rot, v, o, lse, B, T, H, Hkv, D, W, scale, stream);
    return st;
}

int attn_bwd_rope(const attn_bf16* q, const attn_bf16* k, const attn_bf16* q_rot, const attn_bf16* k_rot,
                  const attn_bf16* v, const attn_bf16* o, const float* lse, const attn_bf16* dout, attn_bf16* dq,
                  attn_bf16* dk, attn_bf16* dv, void* workspace, size_t ws_bytes, const float* rope_cos,
                  const float* rope_sin, int max_pos, float eps, int B, int T, int H, int Hkv, int D, int W,
                  float scale, void* stream) {
    if (!q || !k || !q_rot || !k_rot || !aligned16(q) || !aligned16(k) || !aligned16(q_rot) || !aligned16(k_rot))
        return ATTN_ERR_INVALID_ARG;
    if (!valid_rope(rope_cos, rope_sin, max_pos, eps)) return ATTN_ERR_INVALID_ARG;
    // dQ', dK' at the rotated inputs, then back through rotate-and-normalise in place
    int st = attn_bwd_gqa(q_rot, k_rot, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, T, H, Hkv, D, W, scale,
                          stream);
    if (st == ATTN_OK)
        st = rope_qknorm_impl(q, dq, dq, nullptr, rope_cos, rope_sin, max_pos, B, T, H, D, eps, true, stream);
    if (st == ATTN_OK)
        st = rope_qknorm_impl(k, dk, dk, nullptr, rope_cos, rope_sin, max_pos, B, T, Hkv, D, eps, true, stream);
    return st;
}

// Workspace: lse*log2(e) and Delta as [B*H, Tp] fp32 rows (Tp = T rounded up to 128).
size_t attn_bwd_workspace_bytes(int B, int T, int H, int D) {
    if (B < 1 || T < 1 || H < 1 || D < 1) return 0;
    const size_t Tp = (size_t(T) + 127) / 128 * 128;
    return 2 * align256(size_t(B) * H * Tp * 4);
}

int attn_bwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o, const float* lse,
                 const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv, void* workspace,
                 size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, T, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (ws_bytes < attn_bwd_workspace_bytes(B, T, H, D)) return ATTN_ERR_WORKSPACE;
    const int n_blk = (T + 127) / 128;
    const long long n_items = (long long)n_blk * B * H;
    if (n_items > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    const long long grid = n_items < sm_count() ? n_items : sm_count();   // persistent: one CTA per SM
    CUtensorMap mq, mk, mv, mdo;
    if (!make_bthd_map(&mq, q, B, T, H, D) || !make_bthd_map(&mk, k, B, T, Hkv, D) ||
        !make_bthd_map(&mv, v, B, T, Hkv, D) || !make_bthd_map(&mdo, dout, B, T, H, D))
        return ATTN_ERR_LAUNCH;
    const int Tp = (T + 127) / 128 * 128;
    const size_t row_bytes = align256(size_t(B) * H * Tp * 4);
    float* lse2 = reinterpret_cast<float*>(workspace);
    float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + row_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * T * H;
    const auto* o_b = reinterpret_cast<const __nv_bfloat16*>(o);
    const auto* do_b = reinterpret_cast<const __nv_bfloat16*>(dout);
    if (D == 128)
        swa_bwd_pre_kernel<128><<<grid_for(rows * 16, 256), 256, 0, s>>>(o_b, do_b, lse, lse2, delta, B, T, H, Tp);
    else
        swa_bwd_pre_kernel<64><<<grid_for(rows * 8, 256), 256, 0, s>>>(o_b, do_b, lse, lse2, delta, B, T, H, Tp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_LAUNCH;
    if (g_ev_after_pre) cudaEventRecord(g_ev_after_pre, s);

    BwdParams p;
    p.lse2 = lse2;
    p.delta = delta;
    p.dq = reinterpret_cast<__nv_bfloat16*>(dq);
    p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
    p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
    p.B = B;
    p.T = T;
    p.H = H;
    p.G = H / Hkv;
    p.W = W;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_blk = n_blk;
    p.n_items = int(n_items);
    p.Tp = Tp;
    p.wait_limit = kDefaultWaitLimit;
    // dK, dV (key-stationary, one item per key tile of a K/V head), then dQ (query-stationary, one
    // item per query tile of a query head); each launch draws from its own counter.
    const long long n_items_kv = (long long)n_blk * B * Hkv;
    const long long grid_kv = n_items_kv < sm_count() ? n_items_kv : sm_count();
    p.n_items = int(n_items_kv);
    p.work_slot = next_work_slot();
    if (D == 128) {
        if (!ensure_smem((const void*)swa_bwd_dkdv_kernel<128>, BwdKVCfg<128>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_bwd_dkdv_kernel<128><<<unsigned(grid_kv), BwdKVCfg<128>::THREADS, BwdKVCfg<128>::SMEM, s>>>(mq, mk, mv, mdo, p);
    } else {
        if (!ensure_smem((const void*)swa_bwd_dkdv_kernel<64>, BwdKVCfg<64>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_bwd_dkdv_kernel<64><<<unsigned(grid_kv), BwdKVCfg<64>::THREADS, BwdKVCfg<64>::SMEM, s>>>(mq, mk, mv, mdo, p);
    }
    if (launch_status() != ATTN_OK) return ATTN_ERR_LAUNCH;
    if (g_ev_after_main) cudaEventRecord(g_ev_after_main, s);
    p.n_items = int(n_items);
    p.work_slot = next_work_slot();
    if (D == 128) {
        if (!ensure_smem((const void*)swa_bwd_dq_kernel<128>, BwdQCfg<128>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_bwd_dq_kernel<128><<<unsigned(grid), BwdQCfg<128>::THREADS, BwdQCfg<128>::SMEM, s>>>(mq, mk, mv, mdo, p);
    } else {
        if (!ensure_smem((const void*)swa_bwd_dq_kernel<64>, BwdQCfg<64>::SMEM)) return ATTN_ERR_LAUNCH;
        swa_bwd_dq_kernel<64><<<unsigned(grid), BwdQCfg<64>::THREADS, BwdQCfg<64>::SMEM, s>>>(mq, mk, mv, mdo, p);
    }
    return launch_status();
}

int attn_bwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o, const float* lse,
             const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv, void* workspace, size_t ws_bytes,
             int B, int T, int H, int D, int W, float scale, void* stream) {
    return attn_bwd_gqa(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, T, H, H, D, W, scale, stream);
}

// Decode geometry for H query heads over Hkv K/V heads: query heads per thread, slots per CTA,
// (K/V head, query subgroup) pair groups per sequence.
struct DecGeom {
    int qpt, nsub, chunk, nzg;
};
static DecGeom decode_geom(int H, int Hkv, int D) {
    DecGeom g;
    const int kvg = H / Hkv;
    g.qpt = decode_qpt(kvg);
    g.nsub = (kvg + g.qpt - 1) / g.qpt;
    g.chunk = g.qpt == 1 ? kDecodeChunk : kDecodeChunkGrp;
    const int pairs_per_cta = kDecodeThreads / (D / 8);
    g.nzg = (Hkv * g.nsub + pairs_per_cta - 1) / pairs_per_cta;
    return g;
}

size_t attn_decode_gqa_workspace_bytes(int B, int cap, int H, int Hkv, int D) {
    if (B < 1 || cap < 1 || H < 1 || (D != 64 && D != 128) || !valid_kv_heads(H, Hkv)) return 0;
    const DecGeom g = decode_geom(H, Hkv, D);
    const size_t nsm = size_t((cap + g.chunk - 1) / g.chunk);
    return align256(size_t(B) * g.nzg * 4) + align256(size_t(B) * nsm * H * 2 * 4) +
           align256(size_t(B) * nsm * H * D * 4);
}

size_t attn_decode_workspace_bytes(int B, int cap, int H, int D) {
    return attn_decode_gqa_workspace_bytes(B, cap, H, H, D);
}

static int decode_impl(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                       const int32_t* cache_len, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                       int cap, int H, int Hkv, int D, int W, float scale, const RopeArgs& rope,
                       const attn_bf16* k_new, const attn_bf16* v_new, void* stream) {
    if (!q || !k_cache || !v_cache || !cache_len || !o || !workspace) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cache_len) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, cap, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    if (ws_bytes < attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D)) return ATTN_ERR_WORKSPACE;
    const DecGeom g = decode_geom(H, Hkv, D);
    if (g.nzg > 65535) return ATTN_ERR_UNSUPPORTED;
    const int nsm = (cap + g.chunk - 1) / g.chunk;
    const int span = W < cap ? W : cap;
    DecParams p;
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.kc = reinterpret_cast<const __nv_bfloat16*>(k_cache);
    p.vc = reinterpret_cast<const __nv_bfloat16*>(v_cache);
    p.cache_len = cache_len;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    char* ws = static_cast<char*>(workspace);
    const size_t cnt_bytes = align256(size_t(B) * g.nzg * 4);
    p.counters = reinterpret_cast<int*>(ws);
    p.part_ml = reinterpret_cast<float*>(ws + cnt_bytes);
    p.part_o = reinterpret_cast<float*>(ws + cnt_bytes + align256(size_t(B) * nsm * H * 2 * 4));
    p.B = B;
    p.cap = cap;
    p.H = H;
    p.kv_group = H / Hkv;
    p.nsub = g.nsub;
    p.chunk = g.chunk;
    p.W = W;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.nsplit = (span + g.chunk - 1) / g.chunk;
    p.nsplit_max = nsm;
    p.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
    p.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
    p.kc_out = const_cast<__nv_bfloat16*>(p.kc);   // written only with the prologue (attn_decode_rope)
    p.vc_out = const_cast<__nv_bfloat16*>(p.vc);
    p.rope_cos = rope.cs;
    p.rope_sin = rope.sn;
    p.max_pos = rope.max_pos;
    p.eps = rope.eps;
    const int pairs_per_cta = kDecodeThreads / (D / 8);
    const int threads = ((std::min(Hkv * g.nsub, pairs_per_cta) * (D / 8)) + 31) / 32 * 32;
    dim3 grid(p.nsplit, B, g.nzg);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
#define SWA_DECODE_LAUNCH(DD, QQ)                                      \
    do {                                                               \
        if (rope.cs)                                                   \
            swa_decode_kernel<DD, QQ, true><<<grid, threads, 0, s>>>(p);  \
        else                                                           \
            swa_decode_kernel<DD, QQ, false><<<grid, threads, 0, s>>>(p); \
    } while (0)
    if (D == 128) {
        switch (g.qpt) {
            case 1: SWA_DECODE_LAUNCH(128, 1); break;
            case 2: SWA_DECODE_LAUNCH(128, 2); break;
            case 3: SWA_DECODE_LAUNCH(128, 3); break;
            default: SWA_DECODE_LAUNCH(128, 4); break;
        }
    } else {
        switch (g.qpt) {
            case 1: SWA_DECODE_LAUNCH(64, 1); break;
            case 2: SWA_DECODE_LAUNCH(64, 2); break;
            case 3: SWA_DECODE_LAUNCH(64, 3); break;
            default: SWA_DECODE_LAUNCH(64, 4); break;
        }
    }
#undef SWA_DECODE_LAUNCH
    return launch_status();
}

int attn_decode_gqa(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                    const int32_t* cache_len, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                    int cap, int H, int Hkv, int D, int W, float scale, void* stream) {
    return decode_impl(q, k_cache, v_cache, cache_len, o, lse, workspace, ws_bytes, B, cap, H, Hkv, D, W, scale,
                       RopeArgs{}, nullptr, nullptr, stream);
}

int attn_decode_rope(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                     attn_bf16* v_cache, const int32_t* cache_len, const float* rope_cos, const float* rope_sin,
                     int max_pos, float eps, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                     int cap, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) || !valid_rope(rope_cos, rope_sin, max_pos, eps))
        return ATTN_ERR_INVALID_ARG;
    if (!k_cache || !v_cache || !cache_len || !aligned16(k_cache) || !aligned16(v_cache)) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cache_len) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, cap, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    if (ws_bytes < attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D)) return ATTN_ERR_WORKSPACE;
    RopeArgs r;
    r.cs = rope_cos;
    r.sn = rope_sin;
    r.max_pos = max_pos;
    r.eps = eps;
    // One launch: the decode kernel writes the new token's rotated key and its value into slot
    // cache_len[b] - 1 (in the CTAs that read that slot) and rotates the query in registers.
    return decode_impl(q, k_cache, v_cache, cache_len, o, lse, workspace, ws_bytes, B, cap, H, Hkv, D, W, scale, r,
                       k_new, v_new, stream);
}

int attn_decode(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache, const int32_t* cache_len,
                attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B, int cap, int H, int D, int W,
                float scale, void* stream) {
    return attn_decode_gqa(q, k_cache, v_cache, cache_len, o, lse, workspace, ws_bytes, B, cap, H, H, D, W, scale,
                           stream);
}

int attn_decode_noalloc(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                        const int32_t* cache_len, attn_bf16* o, float* lse, int B, int cap, int H, int D, int W,
                        float scale, void* stream) {
    const size_t need = attn_decode_workspace_bytes(B, cap, H, D);
    if (need == 0) return (D != 64 && D != 128 && B >= 1 && cap >= 1 && H >= 1) ? ATTN_ERR_UNSUPPORTED
                                                                                : ATTN_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
    void* ws = noalloc_scratch();
    if (ws == nullptr) return ATTN_ERR_LAUNCH;
    // The ticket counters at the start of the scratch must be zero when a call begins.
    const size_t counter_bytes = size_t(B) * decode_geom(H, H, D).nzg * 4;
    if (cudaMemsetAsync(ws, 0, counter_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
    return attn_decode(q, k_cache, v_cache, cache_len, o, lse, ws, kNoAllocScratchBytes, B, cap, H, D, W, scale,
                       stream);
}

int attn_bwd_set_profile_events(void* after_pre, void* after_main) {
    g_ev_after_pre = reinterpret_cast<cudaEvent_t>(after_pre);
    g_ev_after_main = reinterpret_cast<cudaEvent_t>(after_main);
    return ATTN_OK;
}

int attn_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_LAUNCH;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, swa::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(swa::g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
    }
    if (v & swa::kStatusCacheOverflow) return ATTN_ERR_CACHE_OVERFLOW;
    if (v & swa::kStatusPositionRange) return ATTN_ERR_POSITION_RANGE;
    return v ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

int attn_selftest_wait_timeout(long long limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > (1LL << 34)) return ATTN_ERR_INVALID_ARG;
    swa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
    return launch_status();
}

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_LAUNCH: return "kernel launch failed";
        case ATTN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case ATTN_ERR_WORKSPACE: return "workspace too small";
        case ATTN_ERR_CACHE_OVERFLOW: return "cache capacity exceeded";
        case ATTN_ERR_POSITION_RANGE: return "token position outside the rotary tables";
        default: return "unknown status";
    }
}

}  // extern "C"
