"""Failure handling on the GPU, without faulting or hanging it.

Every pipeline wait of the library is bounded: the combine kernel waits for each
request's split-KV partitions to announce their partial results, and gives up
after 2 s.  Launching the combine stage alone (no split-KV pass, so no
announcement ever comes: a flag that nothing sets) must end within the bound with
MLA_ERR_TIMEOUT in the workspace status word and nothing written, and the CUDA
context must stay usable: a full decode afterwards matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W
from tests.gpu_helpers import compare, oracle_full, run_gpu, to_device

pytestmark = pytest.mark.gpu

MLA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build
    build.build()


def test_combine_wait_times_out_and_the_context_survives(oracle_mod):
    p = W.make_problem([20000, 7000], s_q=1, h_q=128, seed=301)
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
    assert int(ns[-1].item()) > p.batch, "the case must split its sequences"
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
    o = torch.full((p.batch, p.s_q, p.h_q, 512), 3.0, dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), 3.0, dtype=torch.float32, device="cuda")
    call = mla.DecodeCall(q, kv, bt, sl, p.dv, md, ns, softmax_scale=p.scale, workspace=ws, out=o, lse=lse)
    t0 = time.monotonic()
    call.combine()  # no split-KV pass: its announcements never come
    torch.cuda.synchronize()
    waited = time.monotonic() - t0
    assert mla.read_device_status(ws) == MLA_ERR_TIMEOUT
    assert 1.5 < waited < 30.0, waited
    assert bool((o == 3.0).all()) and bool((lse == 3.0).all()), "a timed-out combine wrote results"
    # the context is intact: a complete decode on a fresh workspace is correct
    o2, lse2, _, _ = run_gpu(p)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o2, lse2, o_ref, lse_ref, p.dtype, "after a timed-out wait"))
