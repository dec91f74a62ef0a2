/*
 * swa_attn.h -- C ABI of the B200 (sm_100a) causal sliding-window attention library.
 *
 * The operation.  nanochat's GPT computes attention once per layer through
 * flash_attn_func(q, k, v, causal=True, window_size=window_size) (apidog guide
 * "Train your own ChatGPT", section 5 "Flash Attention unification"), with a
 * per-layer window that alternates short and long contexts in the "SSSL"
 * pattern (same guide, section 1 "GPT model", architecture features), and it
 * decodes tokens against a KV cache prefilled through flash_attn_with_kvcache
 * (same guide, section 6 "Inference engine", KV cache).  Karpathy's nanochat
 * GPT-2-speedrun post (first page) ranks the Flash Attention 3 kernels, whose
 * window_size keyword makes the alternating patterns possible, among the
 * changes that helped most.
 *
 * Window convention used throughout: query i attends to key j iff
 * i - W < j <= i, so row i has min(i + 1, W) keys; W >= T is full causal.
 * The softmax is exp(scale * <q_i, k_j>) normalised over the band; lse is its
 * natural-log normaliser.
 *
 * Common rules for every entry point:
 *  - Tensors are dense, row-major, and live in device memory (the decode
 *    cache_len array too).  The caller owns every buffer, including
 *    workspaces; the library never allocates device memory and never
 *    synchronises in attn_fwd / attn_bwd / attn_decode.  Work is enqueued on
 *    `stream` (a cudaStream_t; NULL means the legacy default stream).
 *  - bf16 tensors are passed as attn_bf16 (the raw 16-bit pattern).
 *    [B, T, H, D] means element (b, t, h, d) at ((b*T + t)*H + h)*D + d.
 *  - Every pointer must be 16-byte aligned; D must be 64 or 128; B, T, H >= 1;
 *    W >= 1; scale > 0 and finite.  A violation returns ATTN_ERR_INVALID_ARG
 *    (or ATTN_ERR_UNSUPPORTED for an unsupported D) before anything is
 *    launched.  A failed launch returns ATTN_ERR_LAUNCH.
 *  - Outputs are written with round-to-nearest-even to bf16; lse is fp32.
 *  - Stream slots.  The library gives each (device, stream) pair it sees a slot: the
 *    first 63 distinct streams of a device get one of their own, later streams share
 *    slot 0.  A slot holds the work counter that the persistent kernels of attn_fwd,
 *    attn_bwd and attn_prefill draw their work items from, and a status word.  Calls
 *    on one stream run one after another and never collide on their slot; calls on
 *    two streams that share slot 0 must not run at the same time.  A CUDA graph
 *    captured from these calls keeps the slot of the stream it was captured on, so
 *    it must not be replayed while eager calls on that stream (or another replay of
 *    it) are running.
 *  - Device-side waits are bounded.  If one gives up (a condition that
 *    correct use never produces), the kernel stops early and records a flag
 *    that attn_device_status() and attn_poll_device_status() report as
 *    ATTN_ERR_DEVICE_TIMEOUT.  A prefill chunk that does not fit its cache is
 *    reported there as ATTN_ERR_CACHE_OVERFLOW, a token position outside the
 *    rotary tables as ATTN_ERR_POSITION_RANGE.
 */
#ifndef SWA_ATTN_H
#define SWA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t attn_bf16;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1,
    ATTN_ERR_UNSUPPORTED = -2,
    ATTN_ERR_LAUNCH = -3,
    ATTN_ERR_DEVICE_TIMEOUT = -4,
    ATTN_ERR_WORKSPACE = -5,
    ATTN_ERR_CACHE_OVERFLOW = -6,
    ATTN_ERR_POSITION_RANGE = -7
} attn_status;

/*
 * Forward (training / prefill): O and logsumexp.
 *   q, k, v  [B, T, H, D] bf16, read only.
 *   o        [B, T, H, D] bf16, written.
 *   lse      [B, H, T] fp32, written; lse[b,h,i] = ln sum_{j in band(i)} exp(scale <q_i, k_j>).
 *   W        window (>= 1; values >= T mean full causal).
 * Defined by: flash_attn_func(q, k, v, causal=True, window_size=...) in the
 * apidog guide, section 5; the window per layer from section 1 ("SSSL").
 */
int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
             int B, int T, int H, int D, int W, float scale, void* stream);

/*
 * Grouped K/V heads (GQA / MQA): the GPT config's n_kv_head (apidog guide,
 * section 1, "GPT model").  k and v are [B, T, Hkv, D] with Hkv >= 1 dividing H;
 * query head h reads K/V head h / (H / Hkv), so H / Hkv consecutive query heads
 * share one K/V head.  Everything else as attn_fwd; attn_fwd is this call with
 * Hkv = H.  Hkv that does not divide H returns ATTN_ERR_INVALID_ARG.
 */
int attn_fwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
                 int B, int T, int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * Chunked prefill against a KV cache, with append: the engine's
 * flash_attn_with_kvcache(q, k_cache, v_cache, k=k_new, v=v_new, cache_seqlens=...)
 * (apidog guide, section 6 "Inference engine") with the window of attn_fwd.
 *   q             [B, Tn, H, D] bf16: a chunk of Tn new tokens per sequence.
 *   k_new, v_new  [B, Tn, Hkv, D] bf16: their keys and values.
 *   k_cache, v_cache  [B, cap, Hkv, D] bf16, updated in place.
 *   cache_len     [B] int32 in device memory: tokens already cached; the chunk's
 *                 token t of sequence b sits at position cache_len[b] + t.
 *   o             [B, Tn, H, D] bf16, written.   lse  [B, H, Tn] fp32, written.
 * The call first writes k_new / v_new into slots cache_len[b] .. cache_len[b]+Tn-1
 * and zeros the slots after them up to the end of that 128-slot block (slots that
 * hold no token); then query t attends to cached positions p - W < j <= p,
 * p = cache_len[b] + t (the previous tokens and the chunk's own, causally).  It does
 * not change cache_len.  cache_len[b] + Tn must not exceed cap: slots past cap are
 * not written and attn_device_status() then reports ATTN_ERR_CACHE_OVERFLOW (the
 * outputs of that sequence are undefined).  Hkv divides H as in attn_fwd_gqa; cap
 * must be >= Tn.  With every cache_len 0 the result equals attn_fwd_gqa on
 * (q, k_new, v_new); with Tn = 1 it is one decode step with append.
 */
int attn_prefill(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                 attn_bf16* v_cache, const int32_t* cache_len, attn_bf16* o, float* lse, int B, int Tn,
                 int cap, int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * Rotary embedding + QK norm, the prologue of attention in the GPT model (apidog guide,
 * section 1 "GPT model", architecture features: rotary embeddings, QK normalisation; an
 * RMSNorm without learnable parameters).  The pages give no formula; the reading used here:
 * for a head vector x at position pos, the pairs (x[i], x[i + D/2]), i < D/2, are rotated by
 * pos * th_i,  r1 = x1 cos - x2 sin,  r2 = x1 sin + x2 cos  (RoFormer), and
 * y = r / sqrt(mean(r^2) + eps).  cos / sin come from fp32 tables [max_pos, D/2] that the
 * caller owns (row pos, column i = angle pos * th_i); eps >= 0 and finite; max_pos >= 1.
 * A token whose position is outside [0, max_pos) is not written, and attn_device_status()
 * reports ATTN_ERR_POSITION_RANGE.
 */

/* Fills the tables for th_i = base^(-2i/D) (base > 1), angles in double precision.
 *   rope_cos, rope_sin  [max_pos, D/2] fp32, written (D even, any size here). */
int attn_rope_tables(float* rope_cos, float* rope_sin, int max_pos, int D, double base, void* stream);

/* y[b,t,h,:] = rotate-and-normalise x[b,t,h,:] at position pos0[b] + t (pos0 NULL: t).
 *   x, y  [B, T, H, D] bf16 (y may be x: in place).  pos0  [B] int32 in device memory, or NULL. */
int attn_rope_qknorm(const attn_bf16* x, attn_bf16* y, const int32_t* pos0, const float* rope_cos,
                     const float* rope_sin, int max_pos, int B, int T, int H, int D, float eps, void* stream);

/* Backward of attn_rope_qknorm: dx = J^T dy at x (same positions), recomputing the rotation:
 * with r = rope(x) and s = (mean(r^2) + eps)^(-1/2), dr = s dy - (s^3 / D) r (dy . r) and dx
 * is dr rotated back.   x, dy, dx  [B, T, H, D] bf16 (dx may be dy). */
int attn_rope_qknorm_bwd(const attn_bf16* x, const attn_bf16* dy, attn_bf16* dx, const int32_t* pos0,
                         const float* rope_cos, const float* rope_sin, int max_pos, int B, int T, int H, int D,
                         float eps, void* stream);

/*
 * Training forward with the prologue: q_rot = rotate-and-normalise(q), k_rot likewise (token t at
 * position t), then attn_fwd_gqa(q_rot, k_rot, v).  q_rot [B, T, H, D] and k_rot [B, T, Hkv, D]
 * bf16 are written (the caller keeps them for attn_bwd_rope).  The keys go through one
 * rotate-and-normalise pass; the queries are rotated and normalised inside the forward kernel,
 * on each query tile in shared memory, which also writes q_rot.  A position outside the tables is
 * reported as ATTN_ERR_POSITION_RANGE, and the outputs of its token are then undefined.  Other
 * arguments as attn_fwd_gqa and attn_rope_qknorm.
 */
int attn_fwd_rope(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* q_rot, attn_bf16* k_rot,
                  attn_bf16* o, float* lse, const float* rope_cos, const float* rope_sin, int max_pos, float eps,
                  int B, int T, int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * Training backward with the prologue: attn_bwd_gqa at (q_rot, k_rot, v), with dq and dk taken
 * back through rotate-and-normalise at the raw q, k (the rounding of q_rot, k_rot to bf16 passes
 * gradients through unchanged, as a cast does).  The dQ kernel does this for dq in its epilogue,
 * before dq is written; dk goes back through it in one pass, in place, after the attention
 * backward.  dq, dk, dv are the gradients with respect to the raw q, k and v.  Workspace as
 * attn_bwd.
 */
int attn_bwd_rope(const attn_bf16* q, const attn_bf16* k, const attn_bf16* q_rot, const attn_bf16* k_rot,
                  const attn_bf16* v, const attn_bf16* o, const float* lse, const attn_bf16* dout, attn_bf16* dq,
                  attn_bf16* dk, attn_bf16* dv, void* workspace, size_t ws_bytes, const float* rope_cos,
                  const float* rope_sin, int max_pos, float eps, int B, int T, int H, int Hkv, int D, int W,
                  float scale, void* stream);

/* Bytes of workspace attn_prefill_rope needs (the chunk's rotated queries, bf16). */
size_t attn_prefill_rope_workspace_bytes(int B, int Tn, int H, int D);

/*
 * attn_prefill with the prologue: q, k_new are the chunk's queries and keys before rotation and
 * norm.  Token t of sequence b is at position cache_len[b] + t: its key is rotated and normalised
 * on the way into the cache (the append writes the rotated, normalised key), its query inside the
 * forward kernel, which also writes the rotated queries into the workspace (at least
 * attn_prefill_rope_workspace_bytes bytes, 256-byte aligned); the forward runs as in
 * attn_prefill.  Tables and eps as attn_rope_qknorm.
 */
int attn_prefill_rope(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                      attn_bf16* v_cache, const int32_t* cache_len, const float* rope_cos, const float* rope_sin,
                      int max_pos, float eps, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                      int Tn, int cap, int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * One decode step with the prologue and append, in one launch: the new token of sequence b
 * sits in slot cache_len[b] - 1 (its position; cache_len counts it, each in [1, cap]).  Its
 * key k_new [B, Hkv, D] is rotated, normalised and written there with its value v_new
 * [B, Hkv, D] by the decode kernel itself, which also rotates and normalises the query
 * q [B, H, D] in registers and then attends as attn_decode_gqa.  workspace: attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D)
 * bytes, zero-filled before first use (every call leaves it zeroed).  Tables and eps as
 * attn_rope_qknorm.
 */
int attn_decode_rope(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_cache,
                     attn_bf16* v_cache, const int32_t* cache_len, const float* rope_cos, const float* rope_sin,
                     int max_pos, float eps, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes, int B,
                     int cap, int H, int Hkv, int D, int W, float scale, void* stream);

/* Bytes of workspace attn_fwd_fp8 needs (V transposed to [B, Hkv, 128, T rounded up to 16]
 * bytes); 0 for sizes it rejects (D other than 128). */
size_t attn_fwd_fp8_workspace_bytes(int B, int T, int Hkv, int D);

/*
 * FP8 forward.  The pages name FP8 only for linear layers (apidog guide, section 3, mixed
 * precision: --fp8 on H100 and Blackwell); the reading for attention: q [B, T, H, 128] and
 * k, v [B, T, Hkv, 128] hold OCP E4M3 bytes (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits), each with one fp32 descale per (sequence, head): q_descale [B, H], k_descale and
 * v_descale [B, Hkv], the real operand being the e4m3 value times its descale.  o [B, T, H, 128]
 * bf16 and lse [B, H, T] fp32 are the windowed attention of attn_fwd_gqa on those real operands,
 * up to the kernel's rounding of the softmax weights to e4m3 before the P V product (each weight
 * off by at most 2^-4 of itself; lse uses the unrounded weights).  workspace: at least
 * attn_fwd_fp8_workspace_bytes(B, T, Hkv, 128) bytes, 256-byte aligned (V is transposed into it);
 * descale pointers 4-byte aligned.  D other than 128 returns ATTN_ERR_UNSUPPORTED.
 */
int attn_fwd_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v, const float* q_descale,
                 const float* k_descale, const float* v_descale, attn_bf16* o, float* lse, void* workspace,
                 size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W, float scale, void* stream);

/* Bytes of workspace attn_bwd needs: fp32 rows of lse*log2(e) and Delta, [B*H, T rounded up
 * to 128] each (256-byte padded). */
size_t attn_bwd_workspace_bytes(int B, int T, int H, int D);

/*
 * Backward: gradients of sum(dO * O) with respect to q, k, v.
 *   q, k, v, o, dout  [B, T, H, D] bf16 (o and lse are the forward's outputs).
 *   lse               [B, H, T] fp32.
 *   dq, dk, dv        [B, T, H, D] bf16, written.
 *   workspace         device buffer of at least attn_bwd_workspace_bytes(B,T,H,D)
 *                     bytes, 256-byte aligned, contents need not be initialised;
 *                     ws_bytes smaller than required returns ATTN_ERR_WORKSPACE.
 * Probabilities are recomputed from lse.  dK, dV and dQ are each accumulated in fp32
 * on chip (tensor memory) and written once as bf16; no atomics, so results are
 * bitwise reproducible run to run.
 * Defined by: training through flash_attn_func (apidog guide, section 5; the
 * training runs of its "scripts.base_train" walkthrough).
 */
int attn_bwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o,
             const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
             void* workspace, size_t ws_bytes, int B, int T, int H, int D, int W, float scale,
             void* stream);

/*
 * Backward with grouped K/V heads: k, v, dk, dv are [B, T, Hkv, D]; dk and dv of a
 * K/V head are the sums over its H / Hkv query heads.  The workspace is
 * attn_bwd_workspace_bytes(B, T, H, D) (per query head).  attn_bwd is this call
 * with Hkv = H.
 */
int attn_bwd_gqa(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* o,
                 const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
                 void* workspace, size_t ws_bytes, int B, int T, int H, int Hkv, int D, int W,
                 float scale, void* stream);

/* Bytes of workspace attn_decode needs for B sequences of capacity cap (any W); 0 for
 * sizes attn_decode rejects (B, cap or H below 1, D not 64 or 128). */
size_t attn_decode_workspace_bytes(int B, int cap, int H, int D);

/*
 * Single-token decode over a KV cache (split over the cache, then combined).
 *   q          [B, H, D] bf16: the new token's query, which sits at position cache_len[b]-1.
 *   k_cache    [B, cap, H, D] bf16; v_cache likewise.  Slot cache_len[b]-1 already
 *              holds the new token's key and value.  Only slots
 *              max(0, L-W) .. L-1 (L = cache_len[b]) are read.
 *   cache_len  [B] int32 in device memory, each in [1, cap].
 *   o          [B, H, D] bf16, written.   lse  [B, H] fp32, written (may be NULL).
 *   workspace  at least attn_decode_workspace_bytes(B, cap, H, D) bytes, 256-byte
 *              aligned.  It must be zero-filled before its first use; every
 *              call leaves it in that state again.  Concurrent calls must not
 *              share a workspace.
 * Defined by: the engine's KV cache and flash_attn_with_kvcache (apidog guide,
 * section 6 "Inference engine").
 */
int attn_decode(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                const int32_t* cache_len, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes,
                int B, int cap, int H, int D, int W, float scale, void* stream);

/* Bytes of workspace attn_decode_gqa needs (any W); 0 for sizes it rejects (as
 * attn_decode_workspace_bytes, or Hkv not dividing H).  With grouped heads one thread serves
 * several query heads of a K/V head over a shorter run of cache slots, so more partials per
 * query head are kept than attn_decode_workspace_bytes(B, cap, H, D) provides for. */
size_t attn_decode_gqa_workspace_bytes(int B, int cap, int H, int Hkv, int D);

/*
 * Decode with grouped K/V heads: k_cache, v_cache are [B, cap, Hkv, D]; query head h
 * reads cache head h / (H / Hkv).  Each K/V row is loaded once for up to four of the query
 * heads that share it.  workspace: at least attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D)
 * bytes, otherwise as attn_decode.  attn_decode is this call with Hkv = H.
 * Defined by: the engine's KV cache (apidog guide, section 6 "Inference engine") with the
 * grouped K/V heads of the model (same guide, section 1 "GPT model").
 */
int attn_decode_gqa(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                    const int32_t* cache_len, attn_bf16* o, float* lse, void* workspace, size_t ws_bytes,
                    int B, int cap, int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * attn_decode without a caller-provided workspace, for callers that cannot
 * allocate device memory: plugins whose host engine owns a fixed
 * device-memory arena and forbids allocation outside it, and latency-bound
 * token loops where an allocation could block on, or synchronise with, the
 * device.  The paper has no counterpart: this is a deployment convenience.
 *   Arguments as for attn_decode, minus workspace / ws_bytes.
 *   Scratch: a fixed 8 MiB device array inside the library (held by every GPU
 *   that loads it until exit).  Sizes whose attn_decode_workspace_bytes
 *   exceeds 8 MiB return ATTN_ERR_WORKSPACE; unsupported D returns
 *   ATTN_ERR_UNSUPPORTED, other bad sizes ATTN_ERR_INVALID_ARG.
 *   The first call on a device looks up the array's device address (set-up,
 *   with that device current); make that first call before any stream capture.
 *   The decode's ticket counters at the start of the array are zero when the
 *   library loads and every call leaves them zero again; the partials are
 *   rewritten by each call before they are read.  All calls share the one
 *   array: calls that overlap on the GPU (other streams, other threads) race
 *   and must be serialised by the caller.  Calls no cudaMalloc / cudaFree and
 *   no allocating library routine.
 */
int attn_decode_noalloc(const attn_bf16* q, const attn_bf16* k_cache, const attn_bf16* v_cache,
                        const int32_t* cache_len, attn_bf16* o, float* lse, int B, int cap, int H, int D, int W,
                        float scale, void* stream);

/*
 * Profiling aid: when set (non-NULL cudaEvent_t handles), every later
 * attn_bwd call made from this host thread records `after_pre` on its stream
 * right after the Delta / lse launch and `after_main` right after the dK/dV
 * launch (the dQ launch follows it), so a caller that brackets attn_bwd with
 * its own events can time the three launches separately.  Pass NULLs to stop.
 * Nothing else changes; no work is skipped.
 */
int attn_bwd_set_profile_events(void* after_pre, void* after_main);

/*
 * Device-wide status word: returns ATTN_OK, or ATTN_ERR_DEVICE_TIMEOUT if any
 * kernel of this library gave up a bounded wait (or found its shared-memory
 * window unusable and did no work) since the last clear (ATTN_ERR_CACHE_OVERFLOW /
 * ATTN_ERR_POSITION_RANGE for those data errors), on any stream.
 * Synchronises the current device.  `clear` != 0 resets the word and every
 * stream slot's word.
 */
int attn_device_status(int clear);

/*
 * Stream-scoped status: waits for the work already queued on `stream` (that stream
 * only), then reads and clears the status word of the stream's slot (see "Stream
 * slots" above) and returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT, ATTN_ERR_CACHE_OVERFLOW
 * or ATTN_ERR_POSITION_RANGE for what the library's kernels on that stream recorded
 * since the last poll of it (or since attn_device_status(1)).  Work on other streams
 * is neither waited for nor reported, unless they share slot 0 with `stream`.
 * ATTN_ERR_LAUNCH if the read itself fails.
 * Defined by: the engine's decode loop, which keeps issuing token steps on its own
 * stream (apidog guide, section 6 "Inference engine").
 */
int attn_poll_device_status(void* stream);

/*
 * Diagnostic: launches one tiny kernel whose mbarrier wait can never complete,
 * bounded by `limit_cycles` SM clocks, so that the bounded-wait path can be
 * exercised without faulting or hanging the GPU.  Returns the launch status;
 * attn_device_status() and attn_poll_device_status(stream) then report
 * ATTN_ERR_DEVICE_TIMEOUT.
 */
int attn_selftest_wait_timeout(long long limit_cycles, void* stream);

/* Human-readable name of a status code. */
const char* attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SWA_ATTN_H */
