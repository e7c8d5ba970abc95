"""nanochat GPT forward + softcapped cross-entropy on B200 (sm_100a).

The compute path is the C-ABI library `libnc.so` (hand-written CUDA kernels);
`decoder_only_transformer_fwd_b200.nc` is its thin ctypes binding.  Importing
the package does not load the library, so the host-side helpers (`synth`,
`flops`) work on machines without a GPU; the first call into `nc` loads it and
raises if it is missing.
"""
