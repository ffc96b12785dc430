"""Failure detection without a GPU fault: a forward launch told to withhold
one mbarrier arrival must run every dependent wait into its (short) limit,
record NEA_ERR_TIMEOUT, return, and leave the context usable."""
import numpy as np
import pytest

import oracle
from causal_gqa_attention_sm_b200.workloads import custom, make_inputs

pytestmark = pytest.mark.gpu


def test_withheld_arrival_times_out_and_context_survives(cuda_lib):
    import torch

    nea = cuda_lib
    w = custom("timeout", B=1, T=256, Hq=2, Hkv=1, D=64, dtype="f32", seed=77)
    t = {n: x.cuda() for n, x in make_inputs(w).items()}
    assert nea.nea_device_status() == nea.NEA_OK
    prev = nea.nea_set_wait_limit_ns(20_000_000)  # 20 ms per wait
    try:
        nea.nea_debug_inject(1)
        nea.nea_attn_fwd(t["q"], t["k"], t["v"], w.rope_base, w.causal)
        assert nea.nea_device_status() == nea.NEA_ERR_TIMEOUT
        assert nea.nea_device_status() == nea.NEA_OK  # the status word was cleared
    finally:
        nea.nea_set_wait_limit_ns(prev)
    o, lse = nea.nea_attn_fwd(t["q"], t["k"], t["v"], w.rope_base, w.causal)
    torch.cuda.synchronize()
    assert nea.nea_device_status() == nea.NEA_OK
    h = {n: x.double().cpu().numpy() for n, x in make_inputs(w).items()}
    ro, _ = oracle.attn_fwd(h["q"], h["k"], h["v"], w.rope_base, w.causal)
    assert np.abs(o.double().cpu().numpy() - ro).max() < 2e-3
