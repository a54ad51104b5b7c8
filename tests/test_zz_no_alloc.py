"""flexq_linear_static_scratch, the linear layer for callers that cannot
allocate device memory (for example a plug-in that its host framework hands
only input and output buffers), keeps its K-split partial sums in a fixed
array inside the library.  Checked here through the C ABI against
flexq_linear with a caller-provided workspace, on two calls in a row (the
second call must clear what the first one left in the shared array), plus the
size limit.  Both entry points run the same kernel with the same K split and
sum the partials in a fixed contributor order, so the outputs must agree bit
for bit (any tolerance would hide a stale partial left in the shared array).
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from gpu_helpers import fq, to_dev, to_host  # noqa: E402

def _inputs(m, n, k, seed):
    rng = np.random.default_rng(seed)
    x = to_dev(rng.standard_normal((m, k)).astype(np.float16))
    w = to_dev((rng.standard_normal((n, k)) * 0.05).astype(np.float16))
    wq = torch.empty(fq.flexq_packed_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
    fq.flexq_quantize_weight_q4(w, n, k, wq)
    bias = to_dev((rng.standard_normal(n) * 0.1).astype(np.float16))
    res = to_dev(rng.standard_normal((m, n)).astype(np.float16))
    return x, wq, bias, res


@pytest.mark.parametrize("m,n,k,splits", [(144, 512, 2048, 8), (32, 1024, 4096, 0)])
def test_static_scratch_matches_workspace_linear_twice(m, n, k, splits):
    x, wq, bias, res = _inputs(m, n, k, m + n)
    epi = fq.EPI_BIAS | fq.EPI_RESIDUAL
    ws_bytes = max(fq.flexq_linear_workspace(m, n, k, 4, splits), 1)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ref = torch.empty(m, n, dtype=torch.float16, device="cuda")
    fq.flexq_linear(x, k, wq, 4, m, n, k, bias, res, n, epi, ref, n, ws, ws_bytes, splits)
    want = to_host(ref)
    assert np.isfinite(want).all()
    for _ in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.float16, device="cuda")
        fq.flexq_linear_static_scratch(x, k, wq, 4, m, n, k, bias, res, n, epi, y, n, splits)
        fq.flexq_device_status()
        got = to_host(y)
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_static_scratch_rejects_oversized_split():
    m, n, k = 600, 8192, 128  # 3 token tiles of 208, 64 feature tiles, 2 K-splits: ~40 MB
    x = torch.zeros(m, k, dtype=torch.float16, device="cuda")
    wq = torch.zeros(fq.flexq_packed_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
    y = torch.zeros(m, n, dtype=torch.float16, device="cuda")
    with pytest.raises(fq.FlexqError) as ei:
        fq.flexq_linear_static_scratch(x, k, wq, 4, m, n, k, None, None, 0, 0, y, n, 2)
    assert ei.value.status == 1 and "static scratch" in str(ei.value)
