"""The device-side timeout path, exercised without faulting the GPU.

With gemm_pair = 2 the MLP down-projection at d24 sizes (M = 8192, N = 1536:
192 tiles of 256 x 256 over 74 CTA pairs) splits the k-blocks of its partial
last wave over all pairs; the pair that finishes such a tile waits, with a
bounded poll, for flags the contributing pairs set.  The test hook makes that
wait expect a generation number the flags never reach and bounds it at 20 ms:
the call must complete, report NC_ERR_TIMEOUT through nc_get_status and leave
the context usable, so that the next normal call gives the same losses as
before.  Nothing else is shortened: the waits on in-flight copies and MMAs
keep their one-second limit and complete normally here."""
import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import nc, synth

pytestmark = pytest.mark.gpu


def test_flag_wait_times_out_and_the_next_call_is_correct():
    import torch
    w = synth.WORKLOADS["d24"]
    B, T = w["B"], w["T"]
    # the first block of the d24 stack alone: its last GEMM is the split-tail down-projection
    cfg = nc.nc_init_config(w["depth"], T, "bf16", "SSSL", w["short"], -1)
    cfg.n_layer, cfg.window[0], cfg.backout_layer = 1, T, 0
    cfg.gemm_pair = 2
    assert cfg.n_embd == 1536 and not cfg.has_ve[0]
    p = synth.params(4242, n_layer=1, n_embd=cfg.n_embd, n_head=cfg.n_head, n_kv_head=cfg.n_kv_head,
                     head_dim=cfg.head_dim, vocab=cfg.vocab, vocab_padded=cfg.vocab_padded, ve_layers=[],
                     bf16=True)
    tok = synth.tokens(4242, B, T, cfg.vocab)
    tgt = synth.targets(4242, B, T, cfg.vocab)
    model = nc.NcModel(cfg, p, B * T)
    t, y = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()

    def run():
        loss, _ = model.forward(t, y)
        torch.cuda.synchronize()
        rc, bits = nc.nc_get_status()
        return loss.cpu().numpy(), rc, bits

    before, rc, _ = run()
    assert rc == 0 and np.all(np.isfinite(before))
    try:
        nc.nc_set_flag_wait_test(1, 20.0)
        _, rc, bits = run()
        assert rc == nc.STATUS_CODES["NC_ERR_TIMEOUT"], (rc, bits)
        assert bits & (1 << nc.STATUS_CODES["NC_ERR_TIMEOUT"])
    finally:
        nc.nc_set_flag_wait_test(0, 1000.0)
    after, rc, bits = run()
    assert rc == 0 and bits == 0
    assert np.array_equal(after, before)
