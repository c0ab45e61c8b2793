"""kascade_decode_anchor_static_ws: the decode anchor for callers that cannot
allocate device memory while they run (for example a runtime plugin whose
enqueue step may not allocate, or a serving engine that has given nearly all
device memory to its KV-cache pool).  Its scratch is a fixed array inside the
library, so the caller passes only inputs and outputs.

The GPU test calls it through the C ABI twice in a row, on different inputs
and sizes (the array keeps the first call's contents), and checks each result
against the regular kascade_decode_anchor with caller-provided scratch, within
the tolerances the other parity tests use.  Around the second call it also
checks that the amount of device memory in use does not change.  This file is named to be collected
after the parity tests; it passes alone in a fresh process and after the rest
of the suite."""
import numpy as np
import pytest
import torch

from long_context_emitting_b200 import api, binding, workload
from long_context_emitting_b200.binding import Shape
from _compare import LSE_ABS, assert_attention_close, assert_pooled_close

SCALE = api.default_scale()


def _outputs(cfg, ld, dev):
    out = torch.full((cfg.B, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((cfg.B, cfg.Hq), float("nan"), dtype=torch.float32, device=dev)
    pooled = torch.zeros(cfg.B, cfg.Hkv, ld, dtype=torch.float32, device=dev)
    return out, lse, pooled


def _call_static(lib, cfg, inp, max_T, ld, out, lse, pooled):
    rc = lib.kascade_decode_anchor_static_ws(
        Shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.d), inp["q"].data_ptr(), inp["k"].data_ptr(),
        inp["v"].data_ptr(), inp["kv_off"].data_ptr(), inp["seq_len"].data_ptr(), max_T, SCALE,
        out.data_ptr(), lse.data_ptr(), pooled.data_ptr(), ld,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 0, binding.STATUS_NAMES.get(rc, rc)


@pytest.mark.gpu
def test_static_scratch_decode_anchor_matches_regular_entry_point():
    lib = binding.load()
    dev = torch.device("cuda")
    runs = [
        (workload.scaled(workload.DECODE_4K, name="static_ws_a", B=2, T=None, T_list=(3001, 4096)), 0),
        (workload.scaled(workload.DECODE_4K, name="static_ws_b", B=3, T=None, T_list=(17, 1000, 2500)), 1),
    ]
    for i, (cfg, layer) in enumerate(runs):
        lens = cfg.seq_lens()
        max_T = max(lens)
        ld = (max_T + 3) // 4 * 4
        shape = Shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.d)
        assert lib.kascade_decode_anchor_workspace_bytes(shape, max_T) <= binding.STATIC_SCRATCH_BYTES
        inp = workload.decode_layer(cfg, layer, dev)
        out, lse, pooled = _outputs(cfg, ld, dev)
        torch.cuda.synchronize()
        if i == 0:
            _call_static(lib, cfg, inp, max_T, ld, out, lse, pooled)
        else:
            # The second call, with its inputs and outputs already in place, must not
            # change how much device memory is in use: neither torch's pool nor the
            # device's free bytes move.
            reserved0 = torch.cuda.memory_reserved(dev)
            free0, _ = torch.cuda.mem_get_info(dev)
            _call_static(lib, cfg, inp, max_T, ld, out, lse, pooled)
            torch.cuda.synchronize()
            assert torch.cuda.memory_reserved(dev) == reserved0
            assert torch.cuda.mem_get_info(dev)[0] == free0
        ref_out, ref_lse, ref_pooled = api.decode_anchor(
            inp["q"], inp["k"], inp["v"], inp["kv_off"], inp["seq_len"], max_T, SCALE, cfg.Hkv,
            ld_pooled=ld)
        assert api.device_status() == 0
        assert_attention_close(out.float().cpu().numpy(), ref_out.float().cpu().numpy(),
                               "static-scratch anchor O")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=LSE_ABS, rtol=0)
        for b, T in enumerate(lens):
            assert_pooled_close(pooled[b, :, :T].cpu().numpy(), ref_pooled[b, :, :T].cpu().numpy(),
                                f"static-scratch pooled b={b}")


def test_static_scratch_refuses_oversized_problem_on_host():
    lib = binding.load()
    shape = Shape(16, 32, 8, 128)
    need = lib.kascade_decode_anchor_workspace_bytes(shape, 32768)
    assert need > binding.STATIC_SCRATCH_BYTES
    p = 0x10000  # never dereferenced: the host refuses before any launch
    rc = lib.kascade_decode_anchor_static_ws(shape, p, p, p, p, p, 32768, SCALE, p, p, p, 32768, None)
    assert rc == 3  # KASCADE_ERR_WORKSPACE_TOO_SMALL
    # argument checks come before the size limit, with the regular entry point's codes
    rc = lib.kascade_decode_anchor_static_ws(shape, p, p, p, p, p, 32768, SCALE, p, p, p, 32766, None)
    assert rc == 1  # KASCADE_ERR_INVALID_ARG: ld_pooled < max_T
    rc = lib.kascade_decode_anchor_static_ws(shape, p, p, p, 0, p, 32768, SCALE, p, p, p, 32768, None)
    assert rc == 1  # KASCADE_ERR_INVALID_ARG: NULL kv_off
