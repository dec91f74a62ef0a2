"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances (fixed by the target, written here):
  O      relative L2 <= 5e-3 and max-abs <= 2e-2
  lse    max-abs <= 1e-3
  dQ/dK/dV relative L2 <= 1e-2
Small shapes are compared element by element over the whole output; the
full-size workloads (depth 12 / 24 / 26 shapes, decode batch) are compared on
sampled rows the oracle computes one by one, plus whole-tensor properties.
"""
import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import (oracle_bwd, oracle_decode, oracle_dkv_rows, oracle_dq_rows, oracle_fwd,
                    oracle_fwd_rows, oracle_prefill)

pytestmark = pytest.mark.gpu

O_REL, O_ABS, LSE_ABS, G_REL = 5e-3, 2e-2, 1e-3, 1e-2
GUARD = 64                      # guard elements on each side of every output (a multiple of 16 bytes)
SENTINEL_BF16 = 0x7BAD
SENTINEL_F32 = 0x7F8BADBD     # a float32 NaN pattern; fits in int32


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_sliding_window_b200 import ops as _ops

    _ops.attn_device_status(clear=True)
    return _ops


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class Guarded:
    """An output tensor with sentinel-filled guard bands before and after it."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
        raw = self.buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32)
        raw.fill_(SENTINEL_BF16 if dtype == torch.bfloat16 else SENTINEL_F32)
        self.t = self.buf[GUARD:GUARD + n].view(shape)

    def guards_intact(self) -> bool:
        raw = self.buf.view(torch.int16 if self.buf.dtype == torch.bfloat16 else torch.int32)
        want = SENTINEL_BF16 if self.buf.dtype == torch.bfloat16 else SENTINEL_F32
        return bool((raw[:GUARD] == want).all() and (raw[-GUARD:] == want).all())


def rel_l2(x, ref):
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30))


def run_fwd_bwd(ops, x, W, with_bwd=True):
    B, T, H, D = x["B"], x["T"], x["H"], x["D"]
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    o, lse = Guarded((B, T, H, D), torch.bfloat16), Guarded((B, H, T), torch.float32)
    ops.attn_fwd(q, k, v, o.t, lse.t, W)
    out = {"o": o, "lse": lse}
    if with_bwd:
        do = dev_bf16(x["do"])
        dq, dk, dv = (Guarded((B, T, H, D), torch.bfloat16) for _ in range(3))
        ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device="cuda")
        ops.attn_bwd(q, k, v, o.t, lse.t, do, dq.t, dk.t, dv.t, ws, W)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    for g in out.values():
        assert g.guards_intact(), "write outside an output buffer"
    return {n: host_f64(g.t) for n, g in out.items()}


SMALL = [
    # (B, T, H, D, W): the tiny workload, ragged tails, several tiles, odd heads, degenerate windows
    (1, 128, 2, 64, 128),
    (1, 128, 2, 64, 32),
    (2, 333, 3, 128, 333),
    (2, 333, 3, 128, 100),
    (2, 333, 3, 128, 129),
    (2, 333, 3, 128, 1),
    (1, 300, 2, 64, 10 ** 9),
    (3, 5, 2, 128, 3),
    (1, 1, 1, 128, 1),
    (1, 1, 2, 64, 7),
    (1, 129, 1, 128, 64),
    (1, 640, 1, 128, 256),
    (1, 700, 13, 128, 200),
    (1, 512, 2, 64, 511),
]


@pytest.mark.parametrize("B,T,H,D,W", SMALL)
def test_small_shapes_match_oracle_elementwise(ops, B, T, H, D, W):
    x = inputs.attention_inputs(B, T, H, D, seed=100 + T + H + (W % 1000))
    got = run_fwd_bwd(ops, x, W)
    o, lse = oracle_fwd(x["q"], x["k"], x["v"], W)
    dq, dk, dv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    assert rel_l2(got["o"], o) <= O_REL
    assert np.max(np.abs(got["o"] - o)) <= O_ABS
    assert np.max(np.abs(got["lse"] - lse)) <= LSE_ABS
    for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
        if np.linalg.norm(ref) == 0:
            # W = 1 (or T = 1): dQ = dK = 0 exactly, since P = 1 and Delta = dP.  The kernel
            # rounds P, O and Delta, leaving a residue of order 1e-6; a relative norm is
            # undefined here, so bound the residue absolutely.
            assert np.max(np.abs(got[name])) <= 1e-4, name
        else:
            assert rel_l2(got[name], ref) <= G_REL, (name, rel_l2(got[name], ref))


FULL = [(name, W) for name in ("d12", "d24", "d26") for W in sorted(set(inputs.WORKLOADS[name]["windows"]))]


def sample_rows(rng, B, T, H, W, n_rand):
    fixed_i = sorted(i for i in {0, 1, W - 1, W, T - 1, T // 2, 127, 128} if 0 <= i < T)
    rows = [(0, 0, i) for i in fixed_i] + [(B - 1, H - 1, i) for i in fixed_i]
    rows += [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(T))) for _ in range(n_rand)]
    return np.array(rows, dtype=np.int64)


@pytest.mark.parametrize("name,W", FULL)
def test_full_size_workloads_sampled(ops, name, W):
    cfg = inputs.WORKLOADS[name]
    B, T, H, D = cfg["B"], cfg["T"], cfg["H"], cfg["D"]
    x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"], peaky=cfg["peaky"])
    got = run_fwd_bwd(ops, x, W)
    for n, a in got.items():
        assert np.isfinite(a).all(), n
    rng = np.random.default_rng(W + H)
    rows = sample_rows(rng, B, T, H, W, 24)
    ro, rl = oracle_fwd_rows(x["q"], x["k"], x["v"], W, rows)
    go = np.stack([got["o"][b, i, h] for b, h, i in rows])
    gl = np.array([got["lse"][b, h, i] for b, h, i in rows])
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    rdq = oracle_dq_rows(x["q"], x["k"], x["v"], x["do"], W, rows)
    gdq = np.stack([got["dq"][b, i, h] for b, h, i in rows])
    assert rel_l2(gdq, rdq) <= G_REL
    # key rows across the whole item order: the first head's, the last head's (the last items a
    # CTA draws, after several others) and random ones
    krows = sample_rows(rng, B, T, H, W, 12)
    rdk, rdv = oracle_dkv_rows(x["q"], x["k"], x["v"], x["do"], W, krows)
    gdk = np.stack([got["dk"][b, j, h] for b, h, j in krows])
    gdv = np.stack([got["dv"][b, j, h] for b, h, j in krows])
    assert rel_l2(gdk, rdk) <= G_REL and rel_l2(gdv, rdv) <= G_REL
    # Whole-tensor property: key i is always in the band of query i, so lse_i >= scale <q_i, k_i>.
    qf, kf = inputs.bf16_bits_to_f64(x["q"][0]), inputs.bf16_bits_to_f64(x["k"][0])
    diag = x["scale"] * np.einsum("thd,thd->ht", qf, kf)
    assert np.all(got["lse"][0] >= diag - LSE_ABS)


def run_decode(ops, x, W, workspace=None, nan_outside=False):
    B, cap, H, D = x["B"], x["cap"], x["H"], x["D"]
    kc, vc = x["k_cache"].copy(), x["v_cache"].copy()
    if nan_outside:
        for b, L in enumerate(x["cache_len"]):
            lo = max(0, int(L) - W)
            kc[b, :lo] = vc[b, :lo] = 0x7FC0       # bf16 NaN in slots before the window
            kc[b, L:] = vc[b, L:] = 0x7FC0         # and in slots past the cache length
    cl = torch.from_numpy(x["cache_len"]).cuda()
    o, lse = Guarded((B, H, D), torch.bfloat16), Guarded((B, H), torch.float32)
    ws = workspace if workspace is not None else ops.decode_workspace(B, cap, H, D, "cuda")
    ops.attn_decode(dev_bf16(x["q"]), dev_bf16(kc), dev_bf16(vc), cl, o.t, lse.t, ws, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    assert o.guards_intact() and lse.guards_intact()
    return host_f64(o.t), host_f64(lse.t), kc, vc


def check_decode(got_o, got_l, ref_o, ref_l):
    assert np.isfinite(got_o).all() and np.isfinite(got_l).all()
    assert rel_l2(got_o, ref_o) <= O_REL
    assert np.max(np.abs(got_o - ref_o)) <= O_ABS
    assert np.max(np.abs(got_l - ref_l)) <= LSE_ABS


@pytest.mark.parametrize("W", [2048, 1024])
def test_decode_workload_matches_oracle(ops, W):
    c = inputs.DECODE_WORKLOAD
    x = inputs.decode_inputs(c["B"], c["cap"], c["H"], c["D"], seed=c["seed"])
    go, gl, _, _ = run_decode(ops, x, W)
    ro, rl = oracle_decode(x["q"], x["k_cache"], x["v_cache"], x["cache_len"], W)
    check_decode(go, gl, ro, rl)


@pytest.mark.parametrize("H,D,W", [(12, 128, 2048), (12, 128, 100), (13, 128, 64), (3, 64, 1), (40, 128, 300),
                                   (5, 64, 10 ** 9)])
def test_decode_edge_lengths_never_read_outside_window(ops, H, D, W):
    lens = np.array([1, 2, 127, 128, 129, 2048, 64, 65, 1000, 1999])
    x = inputs.decode_inputs(len(lens), 2048, H, D, seed=H * D + W % 977, cache_len=lens)
    go, gl, kc, vc = run_decode(ops, x, W, nan_outside=True)
    ro, rl = oracle_decode(x["q"], kc, vc, x["cache_len"], W)
    check_decode(go, gl, ro, rl)


def test_decode_workspace_reuse_is_stable(ops):
    x = inputs.decode_inputs(8, 512, 12, 128, seed=5)
    ws = ops.decode_workspace(8, 512, 12, 128, "cuda")
    first = run_decode(ops, x, 300, workspace=ws)
    second = run_decode(ops, x, 300, workspace=ws)
    assert np.array_equal(first[0], second[0]) and np.array_equal(first[1], second[1])
    assert int(ws[:256].view(torch.int32)[:8].abs().sum()) == 0   # ticket counters back at zero


def test_forward_is_deterministic(ops):
    x = inputs.attention_inputs(2, 400, 3, 128, seed=9, with_do=False)
    a = run_fwd_bwd(ops, x, 150, with_bwd=False)
    b = run_fwd_bwd(ops, x, 150, with_bwd=False)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["lse"], b["lse"])


def test_outputs_16_byte_aligned_only(ops):
    """O, dQ, dK, dV at addresses that are 16-byte but not 32-byte aligned: the epilogues fall back
    from 32-byte to 16-byte stores and the results match the oracle as usual."""
    B, T, H, D, W = 1, 300, 2, 128, 100
    x = inputs.attention_inputs(B, T, H, D, seed=12)
    q, k, v, do = (dev_bf16(x[n]) for n in ("q", "k", "v", "do"))
    n = B * T * H * D

    def offset_view():   # 8 bf16 = 16 bytes past a 256-byte aligned allocation
        buf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
        t = buf[8:].view(B, T, H, D)
        assert t.data_ptr() % 32 == 16
        return t

    o, dq, dk, dv = offset_view(), offset_view(), offset_view(), offset_view()
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    ops.attn_fwd(q, k, v, o, lse, W)
    ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device="cuda")
    ops.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, W)
    torch.cuda.synchronize()
    ro, rl = oracle_fwd(x["q"], x["k"], x["v"], W)
    assert rel_l2(host_f64(o), ro) <= O_REL
    rdq, rdk, rdv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    for got, ref in ((dq, rdq), (dk, rdk), (dv, rdv)):
        assert rel_l2(host_f64(got), ref) <= G_REL


def test_concurrent_streams_keep_their_own_work_counters(ops):
    """Forward and backward launches on two streams, interleaved with no synchronisation between
    them: each stream's persistent kernels draw work items from its own counter, so both
    results equal (bit for bit) those of the same calls run one after another."""
    def setup(B, T, H, seed):
        x = inputs.attention_inputs(B, T, H, 128, seed=seed)
        t = {n: dev_bf16(x[n]) for n in ("q", "k", "v", "do")}
        t["o"], t["dq"], t["dk"], t["dv"] = (torch.empty_like(t["q"]) for _ in range(4))
        t["lse"] = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
        t["ws"] = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, 128), dtype=torch.uint8, device="cuda")
        return t

    def run(t, W, stream=None):
        ops.attn_fwd(t["q"], t["k"], t["v"], t["o"], t["lse"], W, stream=stream)
        ops.attn_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"], t["dq"], t["dk"], t["dv"], t["ws"], W,
                     stream=stream)

    ta, tb = setup(2, 1024, 40, 31), setup(1, 700, 24, 32)   # several items per CTA in each launch
    run(ta, 256)
    run(tb, 1000)
    torch.cuda.synchronize()
    ref = {k: {n: t[n].clone() for n in ("o", "lse", "dq", "dk", "dv")} for k, t in (("a", ta), ("b", tb))}
    for t in (ta, tb):
        for n in ("o", "lse", "dq", "dk", "dv"):
            t[n].zero_()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    sa.wait_stream(torch.cuda.current_stream())
    sb.wait_stream(torch.cuda.current_stream())
    for _ in range(3):
        with torch.cuda.stream(sa):
            run(ta, 256, stream=sa)
        with torch.cuda.stream(sb):
            run(tb, 1000, stream=sb)
    torch.cuda.synchronize()
    assert ops.attn_poll_device_status(sa) == 0 and ops.attn_poll_device_status(sb) == 0
    for k, t in (("a", ta), ("b", tb)):
        for n in ("o", "lse", "dq", "dk", "dv"):
            assert torch.equal(t[n], ref[k][n]), (k, n)


def test_bounded_wait_reports_timeout_without_hanging(ops):
    assert ops.attn_device_status(clear=True) == 0
    assert ops.attn_selftest_wait_timeout(200_000) == 0
    assert ops.attn_device_status(clear=True) == -4       # ATTN_ERR_DEVICE_TIMEOUT
    assert ops.attn_device_status(clear=True) == 0
    # The context is still usable afterwards.
    x = inputs.attention_inputs(1, 64, 1, 64, seed=3, with_do=False)
    got = run_fwd_bwd(ops, x, 16, with_bwd=False)
    o, _ = oracle_fwd(x["q"], x["k"], x["v"], 16)
    assert rel_l2(got["o"], o) <= O_REL


def test_stream_poll_reports_only_that_streams_timeout(ops):
    """attn_poll_device_status(stream): a timeout recorded by a kernel on stream A is reported by
    A's poll (and cleared by it), not by the poll of another stream B; the device-wide word still
    sees it."""
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    assert ops.attn_device_status(clear=True) == 0
    assert ops.attn_poll_device_status(a) == 0 and ops.attn_poll_device_status(b) == 0
    assert ops.attn_selftest_wait_timeout(200_000, stream=a) == 0
    # B's own work, a real forward, is clean and reported clean.
    x = inputs.attention_inputs(1, 200, 2, 64, seed=5, with_do=False)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 200), dtype=torch.float32, device="cuda")
    b.wait_stream(torch.cuda.current_stream())            # the inputs were written on the current stream
    with torch.cuda.stream(b):
        ops.attn_fwd(q, k, v, o, lse, 64, stream=b)
    assert ops.attn_poll_device_status(b) == 0
    assert ops.attn_poll_device_status(a) == -4            # ATTN_ERR_DEVICE_TIMEOUT, read and cleared
    assert ops.attn_poll_device_status(a) == 0
    assert ops.attn_device_status(clear=True) == -4        # the device-wide word saw it too
    assert ops.attn_device_status(clear=True) == 0
    ro, _ = oracle_fwd(x["q"], x["k"], x["v"], 64)
    assert rel_l2(host_f64(o), ro) <= O_REL


# ---------------------------------------------------------------------------
# Grouped K/V heads (the GPT config's n_kv_head): K, V, dK, dV and the caches carry Hkv heads.
# ---------------------------------------------------------------------------
GQA_SMALL = [
    # (B, T, H, Hkv, D, W)
    (1, 333, 4, 2, 128, 100),
    (2, 300, 6, 1, 64, 10 ** 9),    # one K/V head for all query heads
    (1, 640, 8, 4, 128, 129),
    (2, 257, 6, 3, 128, 1),
]


def grouped_inputs(B, T, H, Hkv, D, seed):
    x = inputs.attention_inputs(B, T, H, D, seed=seed)
    x["k"] = np.ascontiguousarray(x["k"][:, :, :Hkv])
    x["v"] = np.ascontiguousarray(x["v"][:, :, :Hkv])
    return x


@pytest.mark.parametrize("B,T,H,Hkv,D,W", GQA_SMALL)
def test_grouped_kv_heads_match_oracle(ops, B, T, H, Hkv, D, W):
    x = grouped_inputs(B, T, H, Hkv, D, seed=500 + T + H)
    q, k, v, do = (dev_bf16(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = Guarded((B, T, H, D), torch.bfloat16), Guarded((B, H, T), torch.float32)
    dq = Guarded((B, T, H, D), torch.bfloat16)
    dk, dv = Guarded((B, T, Hkv, D), torch.bfloat16), Guarded((B, T, Hkv, D), torch.bfloat16)
    ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device="cuda")
    ops.attn_fwd(q, k, v, o.t, lse.t, W)
    ops.attn_bwd(q, k, v, o.t, lse.t, do, dq.t, dk.t, dv.t, ws, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    for g in (o, lse, dq, dk, dv):
        assert g.guards_intact(), "write outside an output buffer"
    ro, rl = oracle_fwd(x["q"], x["k"], x["v"], W)
    rdq, rdk, rdv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    go, gl = host_f64(o.t), host_f64(lse.t)
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    if W == 1:   # dQ = dK = 0 exactly (each row's only key is its own): bound the rounding residue
        assert np.max(np.abs(host_f64(dq.t))) <= 1e-4 and np.max(np.abs(host_f64(dk.t))) <= 1e-4
    else:
        assert rel_l2(host_f64(dq.t), rdq) <= G_REL and rel_l2(host_f64(dk.t), rdk) <= G_REL
    assert rel_l2(host_f64(dv.t), rdv) <= G_REL


# (H, Hkv, D): query heads per thread 3, 4 (two subgroups), 3 (two subgroups), 4 with a ragged
# subgroup of 1, 2, 4 with a ragged subgroup of 3
@pytest.mark.parametrize("H,Hkv,D", [(12, 4, 128), (8, 1, 128), (12, 2, 128), (10, 2, 128), (4, 2, 64), (14, 2, 64)])
def test_grouped_kv_heads_decode(ops, H, Hkv, D):
    B, cap, W = 6, 300, 150
    x = inputs.decode_inputs(B, cap, H, D, seed=H + Hkv + D, cache_len=np.array([1, 64, 149, 151, 300, 233]))
    kc = np.ascontiguousarray(x["k_cache"][:, :, :Hkv])
    vc = np.ascontiguousarray(x["v_cache"][:, :, :Hkv])
    for b, L in enumerate(x["cache_len"]):   # NaN in every slot outside the window: never read
        lo = max(0, int(L) - W)
        kc[b, :lo] = vc[b, :lo] = 0x7FC0
        kc[b, L:] = vc[b, L:] = 0x7FC0
    cl = torch.from_numpy(x["cache_len"]).cuda()
    o, lse = Guarded((B, H, D), torch.bfloat16), Guarded((B, H), torch.float32)
    ws = ops.decode_workspace(B, cap, H, D, "cuda", Hkv=Hkv)
    for _ in range(2):   # the second call checks that the first left the workspace zeroed
        ops.attn_decode(dev_bf16(x["q"]), dev_bf16(kc), dev_bf16(vc), cl, o.t, lse.t, ws, W)
        torch.cuda.synchronize()
        assert ops.attn_device_status(clear=True) == 0
        assert o.guards_intact() and lse.guards_intact()
        ro, rl = oracle_decode(x["q"], kc, vc, x["cache_len"], W)
        check_decode(host_f64(o.t), host_f64(lse.t), ro, rl)


@pytest.mark.parametrize("W", [2048, 1024])
def test_grouped_kv_heads_decode_workload(ops, W):
    """The decode workload with 4 K/V heads for its 12 query heads."""
    c = inputs.DECODE_WORKLOAD
    x = inputs.decode_inputs(c["B"], c["cap"], c["H"], c["D"], seed=c["seed"])
    kc = np.ascontiguousarray(x["k_cache"][:, :, :4])
    vc = np.ascontiguousarray(x["v_cache"][:, :, :4])
    cl = torch.from_numpy(x["cache_len"]).cuda()
    o, lse = ops.decode(dev_bf16(x["q"]), dev_bf16(kc), dev_bf16(vc), cl, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl = oracle_decode(x["q"], kc, vc, x["cache_len"], W)
    check_decode(host_f64(o), host_f64(lse), ro, rl)


def test_grouped_decode_rejects_a_short_workspace(ops):
    """A workspace below attn_decode_gqa_workspace_bytes is rejected before any launch."""
    B, cap, H, Hkv, D = 2, 300, 12, 4, 128
    x = inputs.decode_inputs(B, cap, H, D, seed=5, cache_len=np.array([10, 300]))
    kc = dev_bf16(np.ascontiguousarray(x["k_cache"][:, :, :Hkv]))
    vc = dev_bf16(np.ascontiguousarray(x["v_cache"][:, :, :Hkv]))
    cl = torch.from_numpy(x["cache_len"]).cuda()
    o = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    need = ops.attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D)
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.AttnError):
        ops.attn_decode(dev_bf16(x["q"]), kc, vc, cl, o, lse, ws, 100)


# ---------------------------------------------------------------------------
# Chunked prefill with append against a KV cache.
# ---------------------------------------------------------------------------
NAN_BF16 = 0x7FC0

PREFILL = [
    # (B, Tn, cap, H, Hkv, D, W, cache_len before the chunk)
    (3, 77, 700, 4, 2, 128, 129, (0, 5, 600)),
    (2, 300, 1024, 4, 4, 128, 10 ** 9, (0, 700)),
    (2, 1, 300, 8, 2, 128, 64, (0, 299)),
    (2, 256, 640, 2, 2, 64, 100, (128, 300)),
]


@pytest.mark.parametrize("B,Tn,cap,H,Hkv,D,W,lens", PREFILL)
def test_prefill_matches_oracle_and_appends(ops, B, Tn, cap, H, Hkv, D, W, lens):
    L = np.array(lens, dtype=np.int32)
    x = inputs.attention_inputs(B, Tn, H, D, seed=700 + Tn + cap)
    c = inputs.decode_inputs(B, cap, Hkv, D, seed=701 + Tn)
    kn, vn = (np.ascontiguousarray(x[n][:, :, :Hkv]) for n in ("k", "v"))
    kc, vc = c["k_cache"].copy(), c["v_cache"].copy()
    for b in range(B):   # slots that hold no token: a read that reached P*V would poison the output
        kc[b, L[b] + Tn:] = NAN_BF16
        vc[b, L[b] + Tn:] = NAN_BF16
    dkc, dvc = dev_bf16(kc), dev_bf16(vc)
    o, lse = ops.prefill(dev_bf16(x["q"]), dev_bf16(kn), dev_bf16(vn), dkc, dvc, torch.from_numpy(L).cuda(), W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl, rkc, rvc = oracle_prefill(x["q"], kn, vn, kc, vc, L, W)
    go, gl = host_f64(o), host_f64(lse)
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    got_k = dkc.cpu().view(torch.int16).numpy().view(np.uint16)
    got_v = dvc.cpu().view(torch.int16).numpy().view(np.uint16)
    for b in range(B):
        n = int(L[b]) + Tn
        end = min(cap, (n + 127) // 128 * 128)
        np.testing.assert_array_equal(got_k[b, :n], rkc[b, :n])   # prefix untouched, chunk appended
        np.testing.assert_array_equal(got_v[b, :n], rvc[b, :n])
        assert not got_k[b, n:end].any() and not got_v[b, n:end].any()   # rest of the 128-slot block zeroed
        np.testing.assert_array_equal(got_k[b, end:], kc[b, end:])      # beyond it untouched
        np.testing.assert_array_equal(got_v[b, end:], vc[b, end:])


def test_prefill_overflow_is_reported_and_stays_in_bounds(ops):
    B, Tn, cap, H, D, W = 2, 64, 100, 2, 128, 50
    x = inputs.attention_inputs(B, Tn, H, D, seed=9)
    kc, vc = Guarded((B, cap, H, D), torch.bfloat16), Guarded((B, cap, H, D), torch.bfloat16)
    kc.t.zero_()
    vc.t.zero_()
    L = torch.tensor([0, 50], dtype=torch.int32, device="cuda")   # 50 + 64 > 100 for sequence 1
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    assert ops.attn_device_status(clear=True) == 0
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o, lse = ops.prefill(q, k, v, kc.t, vc.t, L, W, stream=side)
    assert ops.attn_poll_device_status(torch.cuda.current_stream()) == 0   # not this stream's error
    assert ops.attn_poll_device_status(side) == -6      # ATTN_ERR_CACHE_OVERFLOW, on the launching stream
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == -6   # the device-wide word saw it too
    assert kc.guards_intact() and vc.guards_intact()
    ro, rl, _, _ = oracle_prefill(x["q"][:1], x["k"][:1], x["v"][:1], np.zeros((1, cap, H, D), np.uint16),
                                  np.zeros((1, cap, H, D), np.uint16), np.array([0]), W)
    assert rel_l2(host_f64(o[:1]), ro) <= O_REL   # the sequence that fits is unaffected



# ---------------------------------------------------------------------------
# Multi-item persistent launches, compared element by element.  Every persistent kernel runs
# one CTA per SM (148) and draws items from a counter, so the state that runs on from one item
# to the next (K/V ring phases, the Q buffer, the O / dK / dV / dQ accumulators and their
# free barriers, the item ring) is only exercised when a CTA processes several items.  These
# shapes give every CTA at least two items in each kernel:
#   forward items = ceil(T / 256) * B * H, dK/dV items = ceil(T / 128) * B * Hkv,
#   dQ items = ceil(T / 128) * B * H.
# ---------------------------------------------------------------------------
SM_COUNT = 148
MULTI = [
    # (B, T, H, Hkv, D, W)
    (2, 1024, 40, 40, 128, 256),
    (2, 1024, 40, 40, 128, 1024),
    (2, 1000, 40, 40, 64, 300),       # D = 64, ragged last query tile
    (4, 1024, 40, 10, 128, 512),      # grouped K/V heads: 4 query heads per K/V head
    (3, 700, 48, 48, 128, 10 ** 9),   # full causal, ragged tail
]


@pytest.mark.parametrize("B,T,H,Hkv,D,W", MULTI)
def test_multi_item_launches_match_oracle_elementwise(ops, B, T, H, Hkv, D, W):
    n_fwd = -(-T // 256) * B * H
    n_dkdv = -(-T // 128) * B * Hkv
    n_dq = -(-T // 128) * B * H
    assert min(n_fwd, n_dkdv, n_dq) >= 2 * SM_COUNT, "shape too small to give every CTA two items"
    x = inputs.attention_inputs(B, T, H, D, seed=900 + T + H + Hkv + (W % 997))
    x["k"] = np.ascontiguousarray(x["k"][:, :, :Hkv])
    x["v"] = np.ascontiguousarray(x["v"][:, :, :Hkv])
    q, k, v, do = (dev_bf16(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = Guarded((B, T, H, D), torch.bfloat16), Guarded((B, H, T), torch.float32)
    dq = Guarded((B, T, H, D), torch.bfloat16)
    dk, dv = Guarded((B, T, Hkv, D), torch.bfloat16), Guarded((B, T, Hkv, D), torch.bfloat16)
    ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device="cuda")
    ops.attn_fwd(q, k, v, o.t, lse.t, W)
    ops.attn_bwd(q, k, v, o.t, lse.t, do, dq.t, dk.t, dv.t, ws, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    for g in (o, lse, dq, dk, dv):
        assert g.guards_intact(), "write outside an output buffer"
    ro, rl = oracle_fwd(x["q"], x["k"], x["v"], W)
    rdq, rdk, rdv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    go, gl = host_f64(o.t), host_f64(lse.t)
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        g = host_f64(got.t)
        assert rel_l2(g, ref) <= G_REL, (name, rel_l2(g, ref))
    # every (b, h) slice on its own, so that no slice hides behind the whole-tensor norm
    for b in range(B):
        for h in range(H):
            assert rel_l2(go[b, :, h], ro[b, :, h]) <= O_REL, (b, h)
            assert rel_l2(host_f64(dq.t[b, :, h]), rdq[b, :, h]) <= G_REL, (b, h)


def test_multi_item_prefill_matches_oracle(ops):
    """Chunked prefill whose forward launch has B * H * ceil(Tn / 256) = 320 items."""
    B, Tn, cap, H, Hkv, D, W = 8, 512, 2048, 20, 4, 128, 700
    assert B * H * -(-Tn // 256) >= 2 * SM_COUNT
    L = inputs.uniform_int(31, "cache_len", B, 0, cap - Tn).astype(np.int32)
    x = inputs.attention_inputs(B, Tn, H, D, seed=31)
    c = inputs.decode_inputs(B, cap, Hkv, D, seed=32)
    kn, vn = (np.ascontiguousarray(x[n][:, :, :Hkv]) for n in ("k", "v"))
    kc, vc = c["k_cache"].copy(), c["v_cache"].copy()
    for b in range(B):
        kc[b, L[b] + Tn:] = NAN_BF16
        vc[b, L[b] + Tn:] = NAN_BF16
    o, lse = ops.prefill(dev_bf16(x["q"]), dev_bf16(kn), dev_bf16(vn), dev_bf16(kc), dev_bf16(vc),
                         torch.from_numpy(L).cuda(), W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl, _, _ = oracle_prefill(x["q"], kn, vn, kc, vc, L, W)
    go, gl = host_f64(o), host_f64(lse)
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS


def test_depth24_short_window_complete_slices(ops):
    """The depth-24 workload at W = 512, in the launch configuration the benchmark times: four
    complete (b, h) slices spread over the item order (the first head, two middle ones and the
    last, whose items are the last any CTA draws) compared on every row of O, lse and dQ and on
    every key row of dK and dV."""
    cfg = inputs.WORKLOADS["d24"]
    B, T, H, D, W = cfg["B"], cfg["T"], cfg["H"], cfg["D"], 512
    x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"])
    got = run_fwd_bwd(ops, x, W)
    slices = [(0, 0), (B // 3, H // 2), (2 * B // 3, 1), (B - 1, H - 1)]
    rows = np.array([(b, h, i) for b, h in slices for i in range(T)], dtype=np.int64)
    ro, rl = oracle_fwd_rows(x["q"], x["k"], x["v"], W, rows)
    rdq = oracle_dq_rows(x["q"], x["k"], x["v"], x["do"], W, rows)
    rdk, rdv = oracle_dkv_rows(x["q"], x["k"], x["v"], x["do"], W, rows)
    for s, (b, h) in enumerate(slices):
        sl = slice(s * T, (s + 1) * T)
        go, gl = got["o"][b, :, h], got["lse"][b, h]
        assert rel_l2(go, ro[sl]) <= O_REL and np.max(np.abs(go - ro[sl])) <= O_ABS, (b, h)
        assert np.max(np.abs(gl - rl[sl])) <= LSE_ABS, (b, h)
        assert rel_l2(got["dq"][b, :, h], rdq[sl]) <= G_REL, (b, h)
        assert rel_l2(got["dk"][b, :, h], rdk[sl]) <= G_REL, (b, h)
        assert rel_l2(got["dv"][b, :, h], rdv[sl]) <= G_REL, (b, h)
