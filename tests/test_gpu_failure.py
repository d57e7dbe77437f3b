"""Failure paths, exercised without any GPU fault.

* Bounded waits: with the layer's hand-off wait limit set below what any
  hand-off between a GEMM's roles takes, the kernels give up on ordinary
  input; ``moe_layer_sync_status`` must report MOE_ERR_TIMEOUT and the next
  forward with the default limit must be correct again (each CTA drained its
  own copies and tensor-core work and freed its tensor memory; the barrier
  rings are rebuilt per launch).
* Allocation failure: the host-side injection hook MOE_TEST_FAIL_ALLOC_AT=n
  makes the n-th device allocation of ``moe_layer_create`` or of one
  ``moe_layer_set_expert_weights`` call fail; the call must return
  MOE_ERR_OOM, leave nothing half-built behind, and destroy must be clean.
"""
import os

import pytest
import torch

import moe_synth as ms
from moe_testlib import assert_parity, make_blocks, make_layer, oracle_forward

pytestmark = pytest.mark.gpu

MOE_OK, MOE_ERR_OOM, MOE_ERR_NOT_LOADED, MOE_ERR_TIMEOUT = 0, 2, 3, 8


@pytest.fixture(scope="module")
def bq():
    from bit_quantized_moe_top_b200 import build
    build.build()
    import bit_quantized_moe_top_b200 as m
    return m


@pytest.mark.parametrize("path", [1, 2])  # MOE_PATH_DECODE, MOE_PATH_PREFILL
def test_wait_limit_timeout_then_recovery(bq, path):
    cfg = ms.make_config("tiny")
    blocks = make_blocks(cfg, "cuda")
    T = 16 if path == 1 else 128
    L = make_layer(cfg, blocks, max_tokens=T)
    L.set_path(path)
    X, logits = ms.make_inputs(cfg, T, "cuda")
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    Y = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == MOE_OK
    assert_parity(Y, ref["Y"], "before")
    # a 1 ns limit: the first hand-off that is not already complete gives up
    L.set_wait_limit(1)
    seen = []
    for _ in range(5):
        L.forward(X, logits, cfg.top_k)
        seen.append(L.sync_status())
        if seen[-1] == MOE_ERR_TIMEOUT:
            break
    assert MOE_ERR_TIMEOUT in seen, seen
    assert set(seen) <= {MOE_OK, MOE_ERR_TIMEOUT}, seen
    # default limit again: the same layer computes the right answer
    L.set_wait_limit(0)
    for _ in range(3):
        Y = L.forward(X, logits, cfg.top_k)
        assert L.sync_status() == MOE_OK
        assert_parity(Y, ref["Y"], "after")
    L.close()


def _count_allocs(bq, fn):
    """Smallest n for which injection at n no longer fails the call."""
    n = 1
    while True:
        os.environ["MOE_TEST_FAIL_ALLOC_AT"] = str(n)
        try:
            st = fn()
        finally:
            del os.environ["MOE_TEST_FAIL_ALLOC_AT"]
        if st != MOE_ERR_OOM:
            return n, st
        n += 1
        assert n < 200


def test_create_alloc_failure_each_index(bq):
    import ctypes
    cfg = ms.make_config("tiny")
    from moe_testlib import descs_of
    descs = descs_of(cfg)
    arr = (bq.ExpertDesc * cfg.E)(*descs)
    lib = bq._lib()
    handles = []

    def create():
        out = ctypes.c_void_p(1234)
        st = lib.moe_layer_create(cfg.E, cfg.K, cfg.N, 16, cfg.top_k, arr, 0, ctypes.byref(out))
        if st == MOE_ERR_OOM:
            assert out.value is None  # nothing half-built is handed out
        else:
            handles.append(out.value)
        return st

    n, st = _count_allocs(bq, create)
    assert st == MOE_OK and n > 10  # every allocation index of create was failed once
    for h in handles:
        lib.moe_layer_destroy(h)
    torch.cuda.synchronize()


@pytest.mark.parametrize("fmt", ["int", "bitplane"])
def test_set_weights_alloc_failure_each_index(bq, fmt):
    if fmt == "int":
        cfg = ms.make_config("tiny")
    else:
        cfg = ms.scaled_config(ms.make_config("dsv3_bitplane"), E=4, K=256, N=512, top_k=2)
    blocks = make_blocks(cfg, "cuda")
    L = make_layer(cfg, {k: v for k, v in blocks.items() if k != (0, 0)}, max_tokens=16)
    blk = blocks[(0, 0)]
    lib = bq._lib()

    def load():
        return lib.moe_layer_set_expert_weights(
            L.handle, 0, 0, blk.codes.data_ptr(), None if blk.scales is None else blk.scales.data_ptr(),
            blk.zeros_or_lut.data_ptr(), None if blk.rank == 0 else blk.A.data_ptr(),
            None if blk.rank == 0 else blk.B.data_ptr(), 1)

    X, logits = ms.make_inputs(cfg, 16, "cuda")
    Y = torch.empty_like(X)
    os.environ["MOE_TEST_FAIL_ALLOC_AT"] = "1"
    try:
        assert load() == MOE_ERR_OOM
    finally:
        del os.environ["MOE_TEST_FAIL_ALLOC_AT"]
    # a block whose load failed is not loaded: the forward refuses to run
    assert lib.moe_layer_forward(L.handle, X.data_ptr(), logits.data_ptr(), 16, cfg.top_k, Y.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream) == MOE_ERR_NOT_LOADED
    n, st = _count_allocs(bq, load)
    assert st == MOE_OK and n >= 3
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    Y = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == MOE_OK
    assert_parity(Y, ref["Y"], "after the failed loads")
    L.close()
