"""GPU: the host-buffer forward (moesq_moe_forward_host) cuts the batch into token
chunks whose uploads, forward and downloads overlap on three streams.  A token's
result depends only on its own row and routing, so the chunked output must equal the
whole-batch device forward bit for bit, at sizes that take one chunk, three (the
last one short) and the most (8), from pinned and from pageable memory."""
import pytest
import torch

import bench
import workloads as W

pytestmark = pytest.mark.gpu

_LIN = {}


def _bench(T):
    cfg = W.CONFIGS["qwen3_30b_a3b"]
    b = bench.Bench(cfg, T, torch.device("cuda", 0), lin=_LIN)
    _LIN.update(b.lin)
    return b


@pytest.mark.parametrize("T,pinned", [(1, True), (5000, True), (16500, True), (5000, False)])
def test_forward_host_chunked_equals_device(T, pinned):
    b = _bench(T)
    dev_out = b.layer.forward(b.x, b.ids, b.w)
    hx, hids, hw = b.x.cpu(), b.ids.cpu(), b.w.cpu()
    h_out = torch.empty((T, b.cfg.H), dtype=torch.bfloat16)
    if pinned:
        hx, hids, hw, h_out = hx.pin_memory(), hids.pin_memory(), hw.pin_memory(), h_out.pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.layer.forward_host(hx, hids, hw, h_out, d_status=status)
    assert int(status.item()) == 0
    assert torch.equal(h_out, dev_out.cpu())
