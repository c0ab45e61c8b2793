"""Host-side size checks of the Python API, on the CPU.

The C ABI trusts the element counts it is given.  api.py therefore checks
every output, index and table tensor against the count the kernels touch
before it calls the library.  Here the device check is patched out and the
library is replaced by a fake that accepts every call, so only those checks
run.  The tests show two things:
- every call the schedules, the paged path and the calibration helpers make
  passes them;
- each check refuses a tensor that is one element short.
No kernel runs.
"""
import numpy as np
import pytest
import torch

from long_context_emitting_b200 import api, paging, workload
from long_context_emitting_b200.schedule import DecodeSchedule, PrefillSchedule


class _FakeLib:
    """Accepts every entry point; the workspace queries ask for 256 bytes."""

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes"):
            return lambda *a: 256
        return lambda *a: 0


def _need_cpu(name, t, dtype):
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@pytest.fixture
def fake(monkeypatch):
    monkeypatch.setattr(api, "_lib", lambda: _FakeLib())
    monkeypatch.setattr(api, "_need_cuda", _need_cpu)
    monkeypatch.setattr(api, "_ws_bytes", lambda ws: ws.numel() * ws.element_size())
    monkeypatch.setattr(api, "_stream", lambda: 0)
    monkeypatch.setattr(api, "k_for_len", lambda n: int(min(max((n + 5) // 10, 128), n)) if n > 0 else 0)


def _small_decode():
    return workload.scaled(workload.DECODE_4K, name="sizes_decode", B=2, T=300)


def test_schedules_pass_the_checks(fake):
    cfg = _small_decode()
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.seq_lens(), (0,), 2, "cpu")
    lay = workload.decode_layer(cfg, 0, "cpu")
    out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16)
    sch.run_anchor(lay, out)
    sch.run_topk()
    sch.run_reuse(lay, workload.head_map(cfg, 1), out)
    half = {n: (t.to(torch.float16) if n in ("q", "k", "v") else t) for n, t in lay.items()}
    sch.run_anchor(half, out.to(torch.float16))

    pc = workload.scaled(workload.PREFILL_16K, name="sizes_prefill", N=256)
    ps = PrefillSchedule(1, pc.Hq, pc.Hkv, pc.N, (0,), 2, "cpu")
    pin = workload.prefill_layer(pc, 0, "cpu")
    pout = torch.empty_like(pin["q"])
    ps.run_anchor(pin, pout)
    ps.run_topk()
    ps.run_reuse(pin, workload.head_map(pc, 1), pout)


def test_paged_and_calibration_pass_the_checks(fake):
    cfg = _small_decode()
    lay = workload.decode_layer(cfg, 0, "cpu")
    ks = [lay["k"][o: o + cfg.Hkv * T * cfg.d].view(cfg.Hkv, T, cfg.d)
          for o, T in zip(lay["offs"], lay["lens"])]
    vs = [lay["v"][o: o + cfg.Hkv * T * cfg.d].view(cfg.Hkv, T, cfg.d)
          for o, T in zip(lay["offs"], lay["lens"])]
    kp, vp, table, _ = paging.to_paged(ks, vs, 64, spare_pages=2)
    api.decode_anchor_paged(lay["q"], kp, vp, table, 64, lay["seq_len"], 300, 0.1, cfg.Hkv)
    idx = torch.zeros(cfg.B, cfg.Hkv, 128, dtype=torch.int32)
    idx_k = torch.full((cfg.B * cfg.Hkv,), 128, dtype=torch.int32)
    hm = torch.arange(cfg.Hkv, dtype=torch.int32)
    api.decode_reuse_paged(lay["q"], kp, vp, table, 64, lay["seq_len"], idx, idx_k, hm, 0.1, cfg.Hkv)

    p = torch.rand(4, 3, 200)
    api.similarity(p[0], p[1], 16)
    api.head_remap(p, p.flip(0), 16)
    api.similarity_matrix(p, 16)


def _short(t):
    return t.reshape(-1)[:-1].clone()


def test_each_check_refuses_a_short_tensor(fake):
    cfg = _small_decode()
    B, Hq, Hkv, d = cfg.B, cfg.Hq, cfg.Hkv, cfg.d
    lay = workload.decode_layer(cfg, 0, "cpu")
    args = dict(q=lay["q"], k=lay["k"], v=lay["v"], kv_off=lay["kv_off"], seq_len=lay["seq_len"])
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq)
    pooled = torch.empty(B, Hkv, 300)
    for bad in ("kv_off", "seq_len"):
        a = dict(args, **{bad: _short(args[bad])})
        with pytest.raises(ValueError, match=bad):
            api.decode_anchor(a["q"], a["k"], a["v"], a["kv_off"], a["seq_len"], 300, 0.1, Hkv)
    for bad, kw in (("out", dict(out=_short(out))), ("lse", dict(lse=_short(lse))),
                    ("pooled", dict(pooled=_short(pooled)))):
        with pytest.raises(ValueError, match=bad):
            api.decode_anchor(lay["q"], lay["k"], lay["v"], lay["kv_off"], lay["seq_len"], 300, 0.1,
                              Hkv, ld_pooled=300, **kw)

    idx = torch.zeros(B, Hkv, 128, dtype=torch.int32)
    idx_k = torch.full((B * Hkv,), 128, dtype=torch.int32)
    hm = torch.arange(Hkv, dtype=torch.int32)
    for bad, a in (("idx_k", (idx, _short(idx_k), hm)), ("head_map", (idx, idx_k, _short(hm)))):
        with pytest.raises(ValueError, match=bad):
            api.decode_reuse(lay["q"], lay["k"], lay["v"], lay["kv_off"], lay["seq_len"], *a, 0.1, Hkv)
    with pytest.raises(ValueError, match="idx"):  # k_max taken from the last dimension
        api.decode_reuse(lay["q"], lay["k"], lay["v"], lay["kv_off"], lay["seq_len"],
                         idx[:1], idx_k, hm, 0.1, Hkv)

    scores = torch.rand(6, 64)
    rl = torch.full((6,), 64, dtype=torch.int32)
    for bad, a in (("row_len", (_short(rl), rl)), ("row_k", (rl, _short(rl)))):
        with pytest.raises(ValueError, match=bad):
            api.topk(scores, *a, 8)
    with pytest.raises(ValueError, match="out"):
        api.topk(scores, rl, rl, 8, out=torch.empty(6 * 8 - 1, dtype=torch.int32))

    pc = workload.scaled(workload.PREFILL_16K, name="sizes_prefill_bad", N=256)
    pin = workload.prefill_layer(pc, 0, "cpu")
    q, k, v = pin["q"], pin["k"], pin["v"]
    with pytest.raises(ValueError, match="k must be"):
        api.prefill_anchor(q, k[:, :, :128].contiguous(), v, 0.1)
    with pytest.raises(ValueError, match="v must"):
        api.prefill_anchor(q, k, v[:, :4].contiguous(), 0.1)
    with pytest.raises(ValueError, match="pooled"):
        api.prefill_anchor(q, k, v, 0.1, pooled=torch.empty(1, 2, pc.Hkv, 255))
    nt = pc.N // 128
    pidx = torch.zeros(1, nt, pc.Hkv, 128, dtype=torch.int32)
    pidx_k = torch.zeros(nt * pc.Hkv, dtype=torch.int32)
    for bad, a in (("idx_k", (pidx, _short(pidx_k), hm)), ("head_map", (pidx, pidx_k, _short(hm)))):
        with pytest.raises(ValueError, match=bad):
            api.prefill_reuse(q, k, v, *a, 0.1)

    ks = [lay["k"][o: o + Hkv * T * d].view(Hkv, T, d) for o, T in zip(lay["offs"], lay["lens"])]
    vs = [lay["v"][o: o + Hkv * T * d].view(Hkv, T, d) for o, T in zip(lay["offs"], lay["lens"])]
    kp, vp, table, _ = paging.to_paged(ks, vs, 64)
    with pytest.raises(ValueError, match="k_pages"):
        api.decode_anchor_paged(lay["q"], kp, vp, table, 32, lay["seq_len"], 300, 0.1, Hkv)
    with pytest.raises(ValueError, match="block_table"):
        api.decode_anchor_paged(lay["q"], kp, vp, table[:1], 64, lay["seq_len"], 300, 0.1, Hkv)
    with pytest.raises(ValueError, match="v_pages"):
        api.decode_anchor_paged(lay["q"], kp, vp[:1], table, 64, lay["seq_len"], 300, 0.1, Hkv)

    p = torch.rand(4, 64)
    rl4 = torch.full((4,), 64, dtype=torch.int32)
    rk4 = torch.full((4,), 8, dtype=torch.int32)
    ia = torch.zeros(4, 8, dtype=torch.int32)
    with pytest.raises(ValueError, match="idx_b"):
        api.similarity_rows(p, rl4, rk4, ia, _short(ia))
    with pytest.raises(ValueError, match="a_row"):
        api.similarity_rows(p, rl4, rk4, ia, ia, b_row=torch.zeros(6, dtype=torch.int32),
                            a_row=torch.zeros(5, dtype=torch.int32))
