"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on the
same seeded inputs.

* Small problems (the oracle finishes in seconds) are compared element by
  element; they span several pages, ragged page tails, several partitions,
  split and unsplit sequences, 1 to 3 row groups, causal masks that leave rows
  empty, empty sequences and NaN in never-visible cache rows.
* The full-size decode workloads (the five configurations and the compute one
  over an FP8 cache) run in the launch configuration the benchmark times (default scheduler partitions); sampled rows are compared one
  by one with the oracle and every row is checked for finiteness.
"""
import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W
from tests.gpu_helpers import compare, oracle_full, oracle_rows, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build
    build.build()


SMALL = {
    "tiny_workload": lambda: W.make_workload("tiny"),
    "compute_like": lambda: W.make_problem([1000, 3000, 64, 65, 1], s_q=1, h_q=128, seed=101),
    "spec_padded_like": lambda: W.make_workload("spec_padded", seqlens=[300, 420, 511, 129, 64, 2]),
    "long_split_like": lambda: W.make_workload("long_split", seqlens=[20000, 7000, 3000, 100]),
    "fp16_norope_like": lambda: W.make_workload("fp16_norope", seqlens=[700, 130, 2000, 55, 1]),
    "rows72_causal": lambda: W.make_problem([333, 64, 5], s_q=3, h_q=24, causal=True, seed=102),
    "rows200": lambda: W.make_problem([900, 77], s_q=2, h_q=100, causal=True, seed=103),
    "rows256_two_groups": lambda: W.make_problem([1500, 640], s_q=2, h_q=128, causal=True, seed=104),
    "rows384_three_groups": lambda: W.make_problem([400, 90], s_q=3, h_q=128, seed=105),
    "one_head": lambda: W.make_problem([5000, 17], s_q=1, h_q=1, seed=106),
    "empty_and_short": lambda: W.make_problem([0, 1, 2, 0, 63, 64], s_q=4, h_q=16, causal=True, seed=107),
    "nan_poison": lambda: W.make_problem([700, 65, 3], s_q=2, h_q=32, causal=True, seed=108, poison=True,
                                         extra_pages=5),
    "fp16_rope": lambda: W.make_problem([999, 1234], s_q=1, h_q=64, dtype=W.FP16, std=0.5, seed=109),
    "bf16_norope": lambda: W.make_problem([999, 300], s_q=2, h_q=64, d_qk=512, causal=True, seed=110),
    "large_logits": lambda: W.make_problem([2000, 700], s_q=1, h_q=128, seed=111, scale=0.3),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_parity_small(oracle_mod, name):
    p = SMALL[name]()
    o, lse, md, ns = run_gpu(p)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, name))


@pytest.mark.parametrize("parts", [1, 2, 3, 7])
def test_parity_few_partitions(oracle_mod, parts):
    # Few partitions: long chunks, many chunks per partition, pipeline wrap-around
    # across chunks, several splits of one sequence.
    p = W.make_problem([2500, 64, 0, 700, 1, 130], s_q=2, h_q=64, causal=True, seed=120 + parts)
    o, lse, md, ns = run_gpu(p, num_parts=parts)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"parts={parts}"))


def test_parity_more_partitions_than_sm_pairs(oracle_mod):
    # A caller's partition count above the SM pairs (clusters run in two waves) and one
    # sequence split more than 96 ways: the combine reads its splits' LSEs past its registers.
    p = W.make_problem([80000, 3000], s_q=1, h_q=128, seed=140)
    o, lse, md, ns = run_gpu(p, num_parts=110)
    assert int(ns[1].item() - ns[0].item()) > 96, "the long sequence must be split more than 96 ways"
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "110 partitions"))


@pytest.mark.parametrize("parts", [1, 2])
def test_parity_leading_empty_chunks(oracle_mod, parts):
    # A partition whose first chunks are empty sequences: the first non-empty
    # chunk's Q, loaded while the kernel sets up, must reach that chunk.
    p = W.make_problem([0, 0, 700, 0, 130, 0], s_q=1, h_q=32, causal=False, seed=130 + parts)
    o, lse, md, ns = run_gpu(p, num_parts=parts)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"leading empty, parts={parts}"))


@pytest.mark.parametrize("name,parts", [("long_split_like", None), ("compute_like", None), ("few_parts", 3)])
def test_two_stage_calls_match_single_call(name, parts):
    # mla_decode_splitkv followed by mla_decode_combine is the same computation as
    # mla_decode_with_kvcache: bit-identical O and LSE.  The cases cover both combine
    # layouts (many splits per virtual batch, and few).
    p = (W.make_problem([2500, 64, 0, 700, 1, 130], s_q=2, h_q=64, causal=True, seed=140)
         if name == "few_parts" else SMALL[name]())
    o1, lse1, md, ns = run_gpu(p, num_parts=parts)
    q, kv, bt, sl = to_device(p)
    call = mla.DecodeCall(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale)
    call.splitkv()
    call.combine()
    torch.cuda.synchronize()
    assert int(ns[-1].item()) > ns.numel() - 1, "the case must split some sequence"
    assert torch.equal(call.out, o1) and torch.equal(call.lse, lse1)


@pytest.mark.parametrize("case", ["few_splits", "many_splits", "not_a_multiple_of_8", "h_q_not_a_multiple_of_8"])
def test_active_heads(oracle_mod, case):
    # Padding heads (queries zero, as a tensor-parallel rank pads its heads) are neither
    # written nor combined; the real heads match the oracle.  A count that is not a
    # multiple of 8 falls back to every head.
    if case == "many_splits":
        p = W.make_problem([20000, 7000], s_q=2, h_q=64, causal=True, active_heads=16, seed=150)
    elif case == "h_q_not_a_multiple_of_8":
        p = W.make_problem([900, 77], s_q=2, h_q=100, causal=True, active_heads=96, seed=151)
    else:
        p = W.make_workload("spec_padded", seqlens=[300, 420, 511, 129, 64, 2])
    active = {"not_a_multiple_of_8": 12, "h_q_not_a_multiple_of_8": 96}.get(case, 16)
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
    o = torch.full((p.batch, p.s_q, p.h_q, 512), 7.0, dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
    mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale,
                               workspace=ws, out=o, lse=lse, active_heads=active)
    torch.cuda.synchronize()
    assert mla.read_device_status(ws) == 0
    if case == "many_splits":
        assert int(ns[-1].item()) >= 4 * p.batch, "the case must split each sequence several times"
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    real = p.h_q if (active % 8 or p.h_q % 8) else active
    print(compare(o[:, :, :real].contiguous(), lse[:, :, :real].contiguous(), o_ref[:, :, :real], lse_ref[:, :, :real],
                  p.dtype, f"active heads {active} ({case})"))
    if real < p.h_q:
        assert bool((o[:, :, real:] == 7.0).all()), "padding heads' O was written"
        assert bool((lse[:, :, real:] == 7.0).all()), "padding heads' LSE was written"


def test_cached_workspace_across_growing_problems():
    # The API's cached workspace grows with the problem; its control block (status word and
    # split / combine counters) must be zero for every call, including after a larger
    # problem has reused bytes that held split partials before.  Each call must equal the
    # same call on a freshly zeroed workspace.
    probs = [W.make_problem([3000, 900, 4100], s_q=1, h_q=128, seed=160),
             W.make_problem([2500, 64, 700, 1, 130, 5000, 3100, 2000], s_q=2, h_q=64, causal=True, seed=161),
             W.make_problem([3000, 900, 4100], s_q=1, h_q=128, seed=160)]
    for p in probs:
        q, kv, bt, sl = to_device(p)
        md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
        assert int(ns[-1].item()) > ns.numel() - 1, "the case must split some sequence"
        o_c, lse_c = mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale)
        ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
        o_f, lse_f = mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale,
                                                workspace=ws)
        torch.cuda.synchronize()
        assert mla.read_device_status(ws) == 0
        assert torch.equal(o_c, o_f) and torch.equal(lse_c, lse_f)
        zb = mla.workspace_zero_bytes(p.batch, p.s_q, p.h_q, 1)
        assert int(ws[:zb].count_nonzero().item()) == 0, "a call must leave the control block zero"


def test_cached_workspace_shrinking_then_growing(oracle_mod):
    # One cached workspace (the API's default) for a large split batch, then a small split
    # batch, then the large batch twice: the small call's split partials must not land on
    # the counters the large call uses, so every call matches the oracle.
    large = W.make_problem([5000, 300, 2200, 64, 4100, 900, 3000, 1500, 7000, 20], s_q=1, h_q=128, seed=165)
    small = W.make_problem([20000, 9000], s_q=1, h_q=128, seed=166)
    for p in (large, small, large, large):
        q, kv, bt, sl = to_device(p)
        md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
        assert int(ns[-1].item()) > ns.numel() - 1, "the case must split some sequence"
        o, lse = mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale)
        torch.cuda.synchronize()
        ws = mla.api.get_workspace(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), q.device,
                                   mla.workspace_zero_bytes(p.batch, p.s_q, p.h_q, 1))
        assert mla.read_device_status(ws, clear=False) == 0
        o_ref, lse_ref = oracle_full(oracle_mod, p)
        print(compare(o, lse, o_ref, lse_ref, p.dtype, f"batch {p.batch} on the cached workspace"))


def test_metadata_kernel_matches_host_schedule():
    rng = np.random.default_rng(7)
    for hpk in (16, 128, 256):
        L = rng.integers(0, 30000, 97).astype(np.int32)
        sl = torch.from_numpy(L).cuda()
        md, ns = mla.get_mla_metadata(sl, hpk, 1)
        md_h, ns_h = mla.get_mla_metadata_host(L, hpk, 1, md.shape[0])
        assert np.array_equal(md.cpu().numpy(), md_h)
        assert np.array_equal(ns.cpu().numpy(), ns_h)


def test_repeat_calls_are_deterministic():
    p = W.make_problem([3000, 2000, 10], s_q=1, h_q=128, seed=130)
    o1, l1, _, _ = run_gpu(p)
    o2, l2, _, _ = run_gpu(p)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_page_permutation_invariance():
    p = W.make_problem([1000, 300], s_q=2, h_q=64, causal=True, seed=131, extra_pages=7)
    o1, l1, _, _ = run_gpu(p)
    perm = np.random.default_rng(1).permutation(p.num_blocks)
    kv2 = np.empty_like(p.kvcache)
    kv2[perm] = p.kvcache
    p.kvcache = kv2
    p.block_table = np.where(p.block_table >= 0, perm[np.maximum(p.block_table, 0)], -1).astype(np.int32)
    o2, l2, _, _ = run_gpu(p)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_block_table_entry_is_reported():
    # The kernel's own bounds check keeps every load inside the cache and
    # records the error in the workspace status word.
    p = W.make_problem([300, 200], s_q=1, h_q=16, seed=132)
    p.block_table[1, 1] = p.num_blocks + 5  # outside the cache
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8,
                     device="cuda")
    mla.flash_mla_with_kvcache(q, kv, bt, sl, 512, md, ns, workspace=ws)
    assert mla.read_device_status(ws, clear=True) == 6
    assert mla.read_device_status(ws) == 0


def test_host_buffers_end_to_end(oracle_mod):
    p = W.make_problem([700, 64], s_q=2, h_q=16, causal=True, seed=133)
    q, kv, bt, sl = (t.cpu().pin_memory() for t in to_device(p))
    md, ns = mla.get_mla_metadata(sl.cuda(), p.s_q * p.h_q, 1)
    o, lse = mla.flash_mla_with_kvcache(q, kv, bt, sl, 512, md.cpu(), ns.cpu(), causal=True)
    assert not o.is_cuda
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "host buffers"))


# ---------------------------------------------------------------- full-size workloads
def _full_size_sample(p, rng_seed=99):
    rows_total = p.batch * p.s_q * p.h_q
    rng = np.random.default_rng(rng_seed)
    return np.unique(np.concatenate([
        rng.choice(rows_total, size=min(48, rows_total), replace=False),
        [0, rows_total - 1],
        # rows of the longest and the shortest sequence
        np.argmax(p.cache_seqlens) * p.s_q * p.h_q + np.arange(min(8, p.s_q * p.h_q)),
        np.argmin(p.cache_seqlens) * p.s_q * p.h_q + np.arange(min(8, p.s_q * p.h_q)),
    ])).astype(np.int64)


def test_parity_full_size_active_heads(oracle_mod):
    # The speculative workload as the benchmark times it: its 16 real heads of 64 declared
    # with active_heads (the padding-head kernel), full size.  Sampled real-head rows match
    # the oracle; the padding heads' O and LSE are left as they were.
    p = W.make_workload("spec_padded")
    assert p.active_heads == 16
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
    o = torch.full((p.batch, p.s_q, p.h_q, 512), 7.0, dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
    mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale,
                               workspace=ws, out=o, lse=lse, active_heads=p.active_heads)
    torch.cuda.synchronize()
    assert mla.read_device_status(ws) == 0
    rows_total = p.batch * p.s_q * p.h_q
    heads = np.arange(rows_total) % p.h_q
    real = heads < p.active_heads
    sample = _full_size_sample(p)
    sample = np.unique(np.concatenate([sample[real[sample]],
                                       np.random.default_rng(98).choice(np.flatnonzero(real), 48, replace=False)]))
    o_ref, lse_ref = oracle_rows(oracle_mod, p, sample)
    idx = torch.from_numpy(sample).cuda()
    print(compare(o.reshape(rows_total, p.dv)[idx], lse.reshape(rows_total)[idx], o_ref, lse_ref, p.dtype,
                  "spec_padded, 16 active heads, sampled"))
    assert bool((o[:, :, p.active_heads:] == 7.0).all()), "padding heads' O was written"
    assert bool((lse[:, :, p.active_heads:] == 7.0).all()), "padding heads' LSE was written"
    assert torch.isfinite(o[:, :, :p.active_heads]).all()
    assert bool(torch.isfinite(lse[:, :, :p.active_heads]).all())

@pytest.mark.parametrize("name", W.WORKLOADS)
def test_parity_full_size_sampled(oracle_mod, name):
    p = W.make_workload(name)
    o, lse, md, ns = run_gpu(p)
    rows_total = p.batch * p.s_q * p.h_q
    sample = _full_size_sample(p)
    o_ref, lse_ref = oracle_rows(oracle_mod, p, sample)
    o_s = o.reshape(rows_total, p.dv)[torch.from_numpy(sample).cuda()]
    l_s = lse.reshape(rows_total)[torch.from_numpy(sample).cuda()]
    print(compare(o_s, l_s, o_ref, lse_ref, p.dtype, f"{name} sampled"))
    # every row: finite, and finite LSE wherever the row sees at least one token
    assert torch.isfinite(o).all()
    vis = torch.from_numpy(np.repeat(p.visible()[:, :, None], p.h_q, axis=2)).cuda()
    assert torch.equal(torch.isfinite(lse), vis > 0)
    if name == "long_split":
        assert int(ns[-1]) > p.batch  # the scheduler split sequences, so the combine kernel ran
