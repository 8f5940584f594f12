"""Failure handling on the GPU, without faulting or hanging it.

Every pipeline wait of the library is bounded.

* The combine kernel waits for each request's split-KV partitions to announce their
  partial results, and gives up after 2 s.  Launching the combine stage alone (no
  split-KV pass, so no announcement ever comes: a flag that nothing sets) must end
  within the bound with MLA_ERR_TIMEOUT in the workspace status word and nothing
  written, and the CUDA context must stay usable: a full decode afterwards matches
  the oracle.
* The split-KV kernel's roles wait on mbarriers.  A test-only build of the same
  sources (its own shared library, next to the product's) never loads one K page of
  partition 0 and bounds every wait at 0.2 s: the MMA warp's wait for that page runs
  out, the cluster winds down (producers let issued copies land, the MMA warp drains
  and tensor memory is freed), MLA_ERR_TIMEOUT is recorded, the aborted request is
  not written, every row the other clusters wrote is correct, and after the status
  word is cleared the product library decodes on the same workspace correctly.
"""
import ctypes
import os
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


WITHHOLD_PAGE = 3                 # page of partition 0's first chunk that the test build never loads
TEST_WAIT_NS = 200_000_000        # the test build's bound on every wait: 0.2 s
SENTINEL = 3.0


@pytest.fixture(scope="module")
def withholding_lib():
    from mla_decode_attention_12_b200 import _lib, build
    out = os.path.join(os.path.dirname(build.LIB), "_mla_decode_test_withhold.so")
    path = build.build(extra=[f"-DMLA_TEST_WITHHOLD_K_PAGE={WITHHOLD_PAGE}", f"-DMLA_WAIT_TIMEOUT_NS={TEST_WAIT_NS}ull"],
                       out=out)
    return _lib.bind(path)


def test_splitkv_wait_times_out_and_the_context_survives(oracle_mod, withholding_lib):
    from mla_decode_attention_12_b200 import _lib
    lib = withholding_lib
    p = W.make_problem([3000, 5000, 700, 64], s_q=1, h_q=128, seed=302)
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1, num_parts=4)
    m0 = md[0].cpu().numpy()
    # partition 0 starts with request 0 and holds more pages of it than the withheld one
    assert m0[0] == 0 and m0[1] == 0 and (m0[2] > 0 or m0[3] > WITHHOLD_PAGE), m0
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
    o = torch.full((p.batch, p.s_q, p.h_q, 512), SENTINEL, dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), SENTINEL, dtype=torch.float32, device="cuda")
    call = mla.DecodeCall(q, kv, bt, sl, p.dv, md, ns, softmax_scale=p.scale, workspace=ws, out=o, lse=lse)
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    t0 = time.monotonic()
    _lib.check(lib.mla_decode_splitkv(*call.args, stream), "mla_decode_splitkv")
    _lib.check(lib.mla_decode_combine(*call.combine_args, stream), "mla_decode_combine")
    torch.cuda.synchronize()
    waited = time.monotonic() - t0
    status = ctypes.c_int(-1)
    _lib.check(lib.mla_read_device_status(ws.data_ptr(), 0, ctypes.byref(status), stream), "mla_read_device_status")
    assert status.value == MLA_ERR_TIMEOUT, status.value
    assert TEST_WAIT_NS * 1e-9 * 0.75 < waited < 10.0, waited
    # request 0 lost a split: none of its rows is written, by the split-KV pass or the combine
    assert bool((o[0] == SENTINEL).all()) and bool((lse[0] == SENTINEL).all())
    # every row another cluster (or a combine that saw all its splits) wrote is correct
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    untouched = ((o == SENTINEL).all(dim=-1) & (lse == SENTINEL)).cpu().numpy()
    written = ~untouched
    assert written[1:].any(), "the clusters that did not wait on the withheld page finished"
    print(compare(o.cpu()[torch.from_numpy(written)], lse.cpu()[torch.from_numpy(written)], o_ref[written],
                  lse_ref[written], p.dtype, "rows written next to an aborted cluster"))
    # clearing the status word (and the counters the aborted call left) makes the workspace usable
    assert mla.read_device_status(ws, clear=True) == MLA_ERR_TIMEOUT
    o2, lse2 = mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, softmax_scale=p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert mla.read_device_status(ws) == 0
    print(compare(o2, lse2, o_ref, lse_ref, p.dtype, "same workspace after the abort"))
