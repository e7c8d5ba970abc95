"""Kernel attributes (the dynamic shared-memory opt-in of the tcgen05 kernels)
are set per device and remembered per (kernel, device).  A forward pass from
a second host thread, whose CUDA device is selected afresh, and another one
after the device is re-selected on the first thread give bit-identical
results (every reduction of the path runs in a fixed order)."""
import threading

import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc
from nc_cases import make_case, run_gpu

pytestmark = pytest.mark.gpu


def test_second_thread_and_reselected_device_give_the_same_loss():
    import torch
    cfg, _, p, tok, tgt = make_case(4, 2, 256, 128, "bf16", 4242)
    B, T = tok.shape
    loss0, _, rc0, model = run_gpu(cfg, p, tok, tgt)
    assert rc0 == 0

    def forward_once():
        torch.cuda.set_device(0)
        loss, _ = model.forward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
        torch.cuda.synchronize()
        return nc.nc_get_status()[0], loss.view(B, T).cpu().numpy()

    out = {}

    def worker():
        try:
            out["result"] = forward_once()
        except Exception as e:  # reported on the main thread
            out["error"] = e

    th = threading.Thread(target=worker)
    th.start()
    th.join(timeout=300)
    assert not th.is_alive()
    assert "error" not in out, out.get("error")
    rc1, loss1 = out["result"]
    assert rc1 == 0
    assert np.array_equal(loss1, loss0)

    rc2, loss2 = forward_once()
    assert rc2 == 0
    assert np.array_equal(loss2, loss0)
