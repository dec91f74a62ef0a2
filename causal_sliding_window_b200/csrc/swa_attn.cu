// swa_attn.cu -- C-ABI entry points of libswa_b200.so (declared in include/swa_attn.h).
//
// Host side only: argument validation, TMA tensor maps, workspace carving and
// kernel launches on the caller's stream.  No allocation, no synchronisation
// (except attn_device_status, which is documented to synchronise).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/swa_attn.h"
#include "bwd.cuh"
#include "decode.cuh"
#include "fwd.cuh"
#include "fwd_fp8.cuh"
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

// Stream slot of a launch: the first kStreamSlots - 1 distinct streams seen on a device get
// slots 1, 2, ... of their own; later streams share slot 0.  A slot names both the work
// counter of the persistent kernels (launches on one stream never overlap, so they can share
// one) and the status word that attn_poll_device_status(stream) reads.
int stream_slot(cudaStream_t s) {
    static std::mutex mu;
    static std::map<std::pair<int, cudaStream_t>, int> slots;
    static int used[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> g(mu);
    auto it = slots.find({dev, s});
    if (it != slots.end()) return it->second;
    const int slot = used[dev] + 1 < kStreamSlots ? ++used[dev] : 0;
    slots[{dev, s}] = slot;
    return slot;
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

__global__ void swa_selftest_wait_kernel(long long limit_cycles, int slot) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag[2];
    const uint32_t a = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(a, 1);
        abort_flag[0] = 0;
        abort_flag[1] = slot;
        fence_barrier_init();
    }
    __syncthreads();
    // Nobody arrives on this barrier: the wait must give up after limit_cycles.
    if (threadIdx.x == 0) mbar_wait(a, 0, abort_flag, limit_cycles, kStatusTimeoutSelftest);
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

}  // extern "C"

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

// Launches the forward kernel over q [B, T, H, D] against k, v [B, Tk, Hkv, D] (Tk = T, or the cache
// capacity with q_offset set: query t of sequence b at position q_offset[b] + t).  With rope.cs set
// the kernel rotates and normalises the queries itself and writes them to q_rot.
static int launch_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
                      const int32_t* q_offset, int B, int T, int Tk, int H, int Hkv, int D, int W, float scale,
                      const RopeArgs& rope, attn_bf16* q_rot, cudaStream_t s) {
    const int n_qblk = (T + 255) / 256;
    const long long n_items = (long long)n_qblk * B * H;
    if (n_items > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    const long long grid = n_items < sm_count() ? n_items : sm_count();   // persistent: one CTA per SM
    CUtensorMap mq, mk, mv, mqr;
    if (!make_bthd_map(&mq, q, B, T, H, D) || !make_bthd_map(&mk, k, B, Tk, Hkv, D) ||
        !make_bthd_map(&mv, v, B, Tk, Hkv, D) || !make_bthd_map(&mqr, q_rot ? q_rot : q, B, T, H, D))
        return ATTN_ERR_LAUNCH;
    FwdParams p;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.T = T;
    p.H = H;
    p.G = H / Hkv;
    p.q_offset = q_offset;
    p.W = W;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_qblk = n_qblk;
    p.n_items = int(n_items);
    p.stream_slot = stream_slot(s);
    p.wait_limit = kDefaultWaitLimit;
    p.rope_cos = rope.cs;
    p.rope_sin = rope.sn;
    p.max_pos = rope.max_pos;
    p.eps = rope.eps;
    p.store_qrot = q_rot != nullptr;
    const bool off = q_offset != nullptr, r = rope.cs != nullptr;
#define SWA_FWD(DD, OO, RR)                                                                                       \
    do {                                                                                                          \
        if (!ensure_smem((const void*)swa_fwd_kernel<DD, OO, RR>, FwdCfg<DD>::SMEM)) return ATTN_ERR_LAUNCH;     \
        swa_fwd_kernel<DD, OO, RR><<<unsigned(grid), FwdCfg<DD>::threads(RR), FwdCfg<DD>::SMEM, s>>>(mq, mk, mv, \
                                                                                                       mqr, p);  \
    } while (0)
    // Windows shorter than the sequence (training) or than the cache (chunked prefill), no prologue:
    // one MMA issuer per query tile and the key tiles walked downwards, so consecutive items overlap
    // at their solo key steps.
#define SWA_FWD_SHORT(DD, OO)                                                                                     \
    do {                                                                                                          \
        if (!ensure_smem((const void*)swa_fwd_short_kernel<DD, OO>, FwdShortCfg<DD>::SMEM)) return ATTN_ERR_LAUNCH; \
        swa_fwd_short_kernel<DD, OO><<<unsigned(grid), FwdShortCfg<DD>::THREADS, FwdShortCfg<DD>::SMEM, s>>>(    \
            mq, mk, mv, p);                                                                                       \
    } while (0)
    const bool short_window = !r && (long long)W < (off ? Tk : T);
    if (short_window) {
        if (D == 128) {
            if (off) SWA_FWD_SHORT(128, true); else SWA_FWD_SHORT(128, false);
        } else {
            if (off) SWA_FWD_SHORT(64, true); else SWA_FWD_SHORT(64, false);
        }
    } else if (D == 128) {
        if (off) {
            if (r) SWA_FWD(128, true, true); else SWA_FWD(128, true, false);
        } else {
            if (r) SWA_FWD(128, false, true); else SWA_FWD(128, false, false);
        }
    } else {
        if (off) {
            if (r) SWA_FWD(64, true, true); else SWA_FWD(64, true, false);
        } else {
            if (r) SWA_FWD(64, false, true); else SWA_FWD(64, false, false);
        }
    }
#undef SWA_FWD
#undef SWA_FWD_SHORT
    return launch_status();
}

static int bwd_impl(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o, const float* lse,
                    const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv, void* workspace,
                    size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, const RopeArgs& rope,
                    const attn_bf16* q_raw, void* stream);

extern "C" {

int attn_fwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B,
                 int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, T, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    return launch_fwd(q, k, v, o, lse, nullptr, B, T, T, H, Hkv, D, W, scale, RopeArgs{}, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B, int T,
             int H, int D, int W, float scale, void* stream) {
    return attn_fwd_gqa(q, k, v, o, lse, B, T, H, H, D, W, scale, stream);
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
    const int slot = stream_slot(s);
#define SWA_APPEND(DD, RR)                                                                                    \
    swa_append_kernel<DD, RR><<<unsigned(blocks), 256, 0, s>>>(kn, vn, kc, vc, cache_len, B, Tn, cap, Hkv, len_off, \
                                                               tail, rope.cs, rope.sn, rope.max_pos, rope.eps, slot)
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
    // 1. append the chunk's K / V (and zero the rest of its last 128-slot block); with RoPE the keys
    // are rotated and normalised on the way in
    if (launch_append(k_new, v_new, k_cache, v_cache, cache_len, B, Tn, cap, Hkv, D, 0, 128, rope, s) != ATTN_OK)
        return ATTN_ERR_LAUNCH;
    // 2. the forward of the chunk's queries at absolute positions cache_len[b] + t over the cache; with
    // RoPE the forward kernel rotates and normalises the queries itself (and keeps them in q_rot)
    return launch_fwd(q, k_cache, v_cache, o, lse, cache_len, B, Tn, cap, H, Hkv, D, W, scale, rope,
                      rope.cs ? q_rot : nullptr, s);
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
    const int slot = stream_slot(s);
#define SWA_ROPE(DD, BB) \
    swa_rope_qknorm_kernel<DD, BB><<<blocks, 256, 0, s>>>(xx, gg, yy, B, T, H, pos0, rope_cos, rope_sin, max_pos, eps, \
                                                          slot)
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
    // The keys go through one rotate-and-normalise pass (the backward reads k_rot too, so it is
    // materialised); the queries are rotated and normalised inside the forward kernel, which also
    // writes q_rot for the backward.
    int st = rope_qknorm_impl(k, nullptr, k_rot, nullptr, rope_cos, rope_sin, max_pos, B, T, Hkv, D, eps, false, stream);
    if (st != ATTN_OK) return st;
    RopeArgs r;
    r.cs = rope_cos;
    r.sn = rope_sin;
    r.max_pos = max_pos;
    r.eps = eps;
    return launch_fwd(q, k_rot, v, o, lse, nullptr, B, T, T, H, Hkv, D, W, scale, r, q_rot,
                      reinterpret_cast<cudaStream_t>(stream));
}

int attn_bwd_rope(const attn_bf16* q, const attn_bf16* k, const attn_bf16* q_rot, const attn_bf16* k_rot,
                  const attn_bf16* v, const attn_bf16* o, const float* lse, const attn_bf16* dout, attn_bf16* dq,
                  attn_bf16* dk, attn_bf16* dv, void* workspace, size_t ws_bytes, const float* rope_cos,
                  const float* rope_sin, int max_pos, float eps, int B, int T, int H, int Hkv, int D, int W,
                  float scale, void* stream) {
    if (!q || !k || !q_rot || !k_rot || !aligned16(q) || !aligned16(k) || !aligned16(q_rot) || !aligned16(k_rot))
        return ATTN_ERR_INVALID_ARG;
    if (!valid_rope(rope_cos, rope_sin, max_pos, eps)) return ATTN_ERR_INVALID_ARG;
    // The attention backward at the rotated inputs; its dQ kernel takes dq back through
    // rotate-and-normalise at the raw q in its epilogue.  dk goes back through it in place, in one
    // pass after the backward.
    RopeArgs r;
    r.cs = rope_cos;
    r.sn = rope_sin;
    r.max_pos = max_pos;
    r.eps = eps;
    int st = bwd_impl(q_rot, k_rot, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, T, H, Hkv, D, W, scale, r, q,
                      stream);
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

}  // extern "C"

// The backward's three launches.  With rope.cs set, q is the rotated, normalised query and the dQ
// kernel takes dq back through that prologue at q_raw (token t at position t) before writing it.
static int bwd_impl(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o, const float* lse,
                    const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv, void* workspace,
                    size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, const RopeArgs& rope,
                    const attn_bf16* q_raw, void* stream) {
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
    p.q_raw = reinterpret_cast<const __nv_bfloat16*>(q_raw);
    p.rope_cos = rope.cs;
    p.rope_sin = rope.sn;
    p.max_pos = rope.max_pos;
    p.eps = rope.eps;
    const bool r = rope.cs != nullptr;
    // dK, dV (key-stationary, one item per key tile of a K/V head), then dQ (query-stationary, one
    // item per query tile of a query head); each launch draws from its own counter.
    const long long n_items_kv = (long long)n_blk * B * Hkv;
    const long long grid_kv = n_items_kv < sm_count() ? n_items_kv : sm_count();
    p.n_items = int(n_items_kv);
    p.stream_slot = stream_slot(s);
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
    p.stream_slot = stream_slot(s);
#define SWA_DQ(DD, RR)                                                                                      \
    do {                                                                                                    \
        if (!ensure_smem((const void*)swa_bwd_dq_kernel<DD, RR>, BwdQCfg<DD>::SMEM)) return ATTN_ERR_LAUNCH; \
        swa_bwd_dq_kernel<DD, RR><<<unsigned(grid), BwdQCfg<DD>::THREADS, BwdQCfg<DD>::SMEM, s>>>(mq, mk, mv,  \
                                                                                                mdo, p);    \
    } while (0)
    if (D == 128) {
        if (r) SWA_DQ(128, true); else SWA_DQ(128, false);
    } else {
        if (r) SWA_DQ(64, true); else SWA_DQ(64, false);
    }
#undef SWA_DQ
    return launch_status();
}

extern "C" {

int attn_bwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o, const float* lse,
                 const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv, void* workspace,
                 size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, T, H, Hkv, D, W, scale, RopeArgs{},
                    nullptr, stream);
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
    p.stream_slot = stream_slot(s);
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

size_t attn_fwd_fp8_workspace_bytes(int B, int T, int Hkv, int D) {
    if (B < 1 || T < 1 || Hkv < 1 || D != 128) return 0;
    const size_t Tp = (size_t(T) + 15) / 16 * 16;
    return align256(size_t(B) * Hkv * 128 * Tp);
}

int attn_fwd_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v, const float* q_descale,
                 const float* k_descale, const float* v_descale, attn_bf16* o, float* lse, void* workspace,
                 size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, void* stream) {
    if (!q || !k || !v || !q_descale || !k_descale || !v_descale || !o || !lse || !workspace)
        return ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, o, lse};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    const void* dsc[] = {q_descale, k_descale, v_descale};
    for (const void* ptr : dsc)
        if ((reinterpret_cast<uintptr_t>(ptr) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_INVALID_ARG;
    if (!valid_common(B, T, H, D, W, scale) || !valid_kv_heads(H, Hkv)) return ATTN_ERR_INVALID_ARG;
    if (D != 128) return ATTN_ERR_UNSUPPORTED;
    if (ws_bytes < attn_fwd_fp8_workspace_bytes(B, T, Hkv, D)) return ATTN_ERR_WORKSPACE;
    const int n_qblk = (T + 255) / 256;
    const long long n_items = (long long)n_qblk * B * H;
    if (n_items > 0x7fffffffLL || B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
    const int Tp = (T + 15) / 16 * 16;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* vt = static_cast<uint8_t*>(workspace);
    // 1. V^T [B, Hkv, 128, Tp]: the P V product reads V as a K-major operand
    swa_fp8_transpose_v_kernel<<<dim3(unsigned((T + 63) / 64), unsigned(Hkv), unsigned(B)), 256, 0, s>>>(v, vt, T, Hkv,
                                                                                                          Tp);
    if (launch_status() != ATTN_OK) return ATTN_ERR_LAUNCH;
    // 2. the forward: 8-bit [B, T, H(kv), 128] maps, one 128 x 128-byte box per tile
    auto enc = encode_fn();
    if (!enc) return ATTN_ERR_LAUNCH;
    auto map8 = [&](CUtensorMap* m, const void* base, cuuint64_t d0, cuuint64_t d1, cuuint64_t d2, cuuint64_t d3,
                    cuuint32_t b0, cuuint32_t b1, cuuint32_t b2) {
        cuuint64_t dims[4] = {d0, d1, d2, d3};
        cuuint64_t strides[3] = {d0, d0 * d1, d0 * d1 * d2};
        cuuint32_t box[4] = {b0, b1, b2, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    CUtensorMap mq, mk, mvt;
    if (!map8(&mq, q, 128, H, T, B, 128, 1, 128) || !map8(&mk, k, 128, Hkv, T, B, 128, 1, 128) ||
        !map8(&mvt, vt, Tp, 128, Hkv, B, 128, 128, 1))
        return ATTN_ERR_LAUNCH;
    Fp8Params p;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.dq = q_descale;
    p.dk = k_descale;
    p.dv = v_descale;
    p.B = B;
    p.T = T;
    p.H = H;
    p.G = H / Hkv;
    p.W = W;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.n_qblk = n_qblk;
    p.n_items = int(n_items);
    p.stream_slot = stream_slot(s);
    p.wait_limit = kDefaultWaitLimit;
    const long long grid = n_items < sm_count() ? n_items : sm_count();
    if (!ensure_smem((const void*)swa_fwd_fp8_kernel, Fp8Cfg::SMEM)) return ATTN_ERR_LAUNCH;
    swa_fwd_fp8_kernel<<<unsigned(grid), Fp8Cfg::THREADS, Fp8Cfg::SMEM, s>>>(mq, mk, mvt, p);
    return launch_status();
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
    // The ticket counters at the start of the scratch must be zero when a call begins: the array
    // starts zeroed, and the last CTA of every (sequence, head group) of a decode launch puts its
    // counter back to zero, so nothing needs clearing here.
    return attn_decode(q, k_cache, v_cache, cache_len, o, lse, ws, kNoAllocScratchBytes, B, cap, H, D, W, scale,
                       stream);
}

int attn_bwd_set_profile_events(void* after_pre, void* after_main) {
    g_ev_after_pre = reinterpret_cast<cudaEvent_t>(after_pre);
    g_ev_after_main = reinterpret_cast<cudaEvent_t>(after_main);
    return ATTN_OK;
}

static int status_code(int v) {
    if (v & swa::kStatusCacheOverflow) return ATTN_ERR_CACHE_OVERFLOW;
    if (v & swa::kStatusPositionRange) return ATTN_ERR_POSITION_RANGE;
    return v ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

int attn_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_LAUNCH;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, swa::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
    if (clear) {
        const int zero = 0;
        static const int zeros[swa::kStreamSlots] = {0};
        if (cudaMemcpyToSymbol(swa::g_attn_status, &zero, sizeof(int)) != cudaSuccess ||
            cudaMemcpyToSymbol(swa::g_stream_status, zeros, sizeof(zeros)) != cudaSuccess)
            return ATTN_ERR_LAUNCH;
    }
    return status_code(v);
}

int attn_poll_device_status(void* stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int slot = stream_slot(s);
    int* word = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&word), swa::g_stream_status) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
    word += slot;
    int v = 0;
    // The read is queued behind the stream's work; the clear behind the read.
    if (cudaMemcpyAsync(&v, word, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(word, 0, sizeof(int), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
    return status_code(v);
}

int attn_selftest_wait_timeout(long long limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > (1LL << 34)) return ATTN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    swa_selftest_wait_kernel<<<1, 32, 0, s>>>(limit_cycles, stream_slot(s));
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
