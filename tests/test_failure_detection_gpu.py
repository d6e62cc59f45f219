"""Failure detection on the GPU without a GPU fault.

Every device-side wait in the library is bounded: a wait that cannot complete
sets LSA_DEV_ERR_TIMEOUT in the device status word and the kernel returns.
These tests make such a wait run out on purpose (an mbarrier that nothing
completes; a flag that nothing sets), with a short limit, and check that the
status is reported, that it is cleared on read, and that the context still
runs the decode path afterwards.  The host-side argument checks are covered
on the CPU by test_abi.py.
"""
import time

import pytest
import torch

import kv_chunk_selection_b200 as lsa
from lsa_testlib import assert_attention_close, cm, f64
import oracle

pytestmark = pytest.mark.gpu
TIMEOUT = 16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_chunk_selection_b200 import build
    build.build()
    lsa.lib()
    lsa.read_device_status()   # start clean


def test_mbarrier_wait_that_cannot_complete_times_out():
    t0 = time.perf_counter()
    lsa.lsa_selftest_bounded_wait(0, None, 20000)          # 20 ms limit
    bits = lsa.read_device_status()
    assert bits & TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert lsa.read_device_status() == 0                    # read clears it


def test_flag_never_set_times_out_and_set_flag_does_not():
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_selftest_bounded_wait(1, flag, 20000)
    assert lsa.read_device_status() & TIMEOUT
    flag.fill_(1)
    lsa.lsa_selftest_bounded_wait(1, flag, 20000)
    assert lsa.read_device_status() == 0


def test_context_usable_after_timeouts():
    lsa.lsa_selftest_bounded_wait(0, None, 5000)
    assert lsa.read_device_status() & TIMEOUT
    n_kept = [3, 40]
    total = sum(n_kept)
    g = torch.Generator(device="cuda").manual_seed(1)
    kb = torch.randn((8, total, 64, 128), generator=g, device="cuda").to(torch.bfloat16)
    vb = torch.randn_like(kb, dtype=torch.float32).to(torch.bfloat16)
    cu = torch.tensor([0, 3, total], dtype=torch.int32, device="cuda")
    q = torch.randn((2, 64, 128), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.empty((2, 64, 128), device="cuda")
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out, lsa.new_attn_workspace(2))
    torch.cuda.synchronize()
    assert lsa.read_device_status() == 0
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), cu.cpu().numpy())
    assert_attention_close(out, ref)


def test_selftest_rejects_bad_arguments():
    with pytest.raises(lsa.LsaError):
        lsa.lsa_selftest_bounded_wait(2, None, 1000)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_selftest_bounded_wait(1, None, 1000)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_selftest_bounded_wait(0, None, 0)
