"""The process-pool runner of the oracle gives the oracle's own result: same
routing, and outputs equal to the sequential forward (same per-expert row
sets, same arithmetic), on integer and bit-plane layers with compensators,
all rows and a row subset, with top-n compensation."""
import numpy as np
import pytest

import moe_synth as ms
import oracle as orc
from moe_testlib import OracleExperts, make_blocks
import oracle_pool


@pytest.mark.parametrize("fmt", ["int", "bitplane"])
@pytest.mark.parametrize("rows,ctn", [(None, 0), ([0, 3, 7, 12], 0), (None, 1)])
def test_pool_forward_equals_oracle(fmt, rows, ctn):
    if fmt == "int":
        cfg = ms.scaled_config(ms.make_config("mixtral_decode", comp_std_mult=10.0), E=6, K=256, N=256, top_k=2)
    else:
        cfg = ms.scaled_config(ms.make_config("dsv3_bitplane", comp_std_mult=10.0), E=6, K=256, N=256, top_k=3)
    blocks = make_blocks(cfg, "cpu")
    X, logits = ms.make_inputs(cfg, 16, "cpu")
    Xn = X.float().numpy().astype(np.float64)
    Ln = logits.numpy()
    ref = orc.moe_forward(Xn, Ln, cfg.top_k, OracleExperts(blocks), cfg.N, rows=rows, comp_top_n=ctn)
    from moe_testlib import _block_job_dict
    got = oracle_pool.forward(Xn, Ln, cfg.top_k, lambda e: {b: _block_job_dict(blocks[(e, b)]) for b in (0, 1)},
                              cfg.N, rows=rows, comp_top_n=ctn, procs=2)
    for key in ("idx", "counts", "offsets", "perm_token", "inv_pos"):
        assert np.array_equal(got[key], ref[key])
    assert np.max(np.abs(got["Y"] - ref["Y"])) <= 1e-12 * np.max(np.abs(ref["Y"]))
