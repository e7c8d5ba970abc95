"""Shared set-up for the GPU parity tests: one seeded parameter set and token
batch feeds both the CUDA path (through the C ABI) and the oracle."""
import numpy as np

from decoder_only_transformer_fwd_b200 import nc, synth
from oracle import nanochat_fwd as O


def make_case(depth, B, T, short, dtype, seed, *, max_T=None, pattern="SSSL", layers=None, n_kv_head=None):
    max_T = T if max_T is None else max_T
    cfg = nc.nc_init_config(depth, max_T, dtype, pattern, short, -1)
    if n_kv_head is not None:
        cfg.n_kv_head = n_kv_head
    ocfg = O.make_config(depth, max_T, short, pattern=pattern, n_kv_head=n_kv_head)
    params = synth.params(seed, n_layer=cfg.n_layer, n_embd=cfg.n_embd, n_head=cfg.n_head,
                          n_kv_head=cfg.n_kv_head, head_dim=cfg.head_dim, vocab=cfg.vocab,
                          vocab_padded=cfg.vocab_padded, ve_layers=ocfg["ve_layers"],
                          bf16=(dtype == "bf16"), layers=layers)
    tok = synth.tokens(seed, B, T, cfg.vocab)
    tgt = synth.targets(seed, B, T, cfg.vocab)
    return cfg, ocfg, params, tok, tgt


def run_gpu(cfg, params, tok, tgt, want_logits=False, max_tokens=None):
    import torch
    B, T = tok.shape
    model = nc.NcModel(cfg, params, max_tokens or B * T)
    t = torch.from_numpy(tok).cuda()
    y = torch.from_numpy(tgt).cuda()
    loss, logits = model.forward(t, y, want_logits=want_logits)
    torch.cuda.synchronize()
    rc, bits = nc.nc_get_status()
    out_logits = None if logits is None else logits.view(B, T, -1).cpu().numpy()
    return loss.view(B, T).cpu().numpy(), out_logits, rc, model
