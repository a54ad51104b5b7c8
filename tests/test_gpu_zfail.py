"""Failure paths on the GPU without faulting it: a bounded device wait that
runs out reports FLEXQ_ERR_TIMEOUT and leaves the context usable; a token id
outside the vocabulary is reported, never dereferenced."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import q64  # noqa: E402
from gpu_helpers import assert_close, fq, to_dev, to_host  # noqa: E402


def _gemm(m=128, n=1024, k=4096):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((m, k)).astype(np.float16)
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float16)
    wd = torch.empty(fq.flexq_packed_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
    fq.flexq_quantize_weight_q4(to_dev(w), n, k, wd)
    y = torch.empty(m, n, dtype=torch.float16, device="cuda")
    xd = to_dev(x)

    def run():
        fq.flexq_linear(xd, k, wd, 4, m, n, k, None, None, 0, 0, y, n, None, 0, 1)

    ref = x.astype(np.float64) @ q64.roundtrip(w).astype(np.float64).T
    return run, y, ref


def test_wait_timeout_is_reported_and_context_survives():
    run, y, ref = _gemm()
    fq.flexq_device_status()
    try:
        fq.flexq_set_wait_limit_ns(1)
        run()
        with pytest.raises(fq.FlexqError) as ei:
            fq.flexq_device_status()
        assert ei.value.status == 4
    finally:
        fq.flexq_set_wait_limit_ns(0)
    run()
    fq.flexq_device_status()
    assert_close(to_host(y), ref, 2e-3)


def test_bad_token_id_is_reported():
    import synth
    from quantized_opt_decode_b200.device_model import DeviceModel, workspace
    p = dict(synth.CONFIGS["tiny"])
    dm = DeviceModel(p, b=1, max_len=6, layers=1)
    prompt = torch.tensor([[1, 2, p["vocab"] + 5, 3]], dtype=torch.int32, device="cuda")
    out = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    ws_n = fq.flexq_generate_workspace(dm.struct, 1, 4, 1)
    ws = workspace(ws_n)
    fq.flexq_generate(dm.struct, prompt, 1, 4, 2, 1, out, ws, ws_n)
    with pytest.raises(fq.FlexqError) as ei:
        fq.flexq_device_status()
    assert ei.value.status == 6
    fq.flexq_device_status()  # cleared
