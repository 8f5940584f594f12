"""Per-phase timeline of the split-KV kernel, from an instrumented copy of the library.

Builds ``_mla_decode_timeline.so`` (the same source compiled with ``-DMLA_TIMELINE``: a few
threads of every CTA write (event, %globaltimer) words into a device array), runs the
split-KV and combine kernels of each workload on the GPU with the L2 flushed before every
launch, reads the events of the last launch and splits each cluster's time into phases:

* start-up: kernel entry -> the first page's logits (barriers, tensor memory, first Q and K);
* streaming: first logits -> last P of each chunk (the page loop);
* transitions: last P of a chunk -> first logits of the next (last P V, output drained from
  tensor memory, then the next chunk's logits; and, on the MMA warp, the next chunk's Q ready);
* last epilogue: last P of the last chunk -> the cluster's exit;
* idle at the end: the cluster's exit -> the last cluster's exit.

Usage: ``python -m mla_decode_attention_12_b200.timeline [--workloads compute,long_split]``
prints a markdown summary (needs a B200).  The product library is not touched.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

import numpy as np

from . import _lib, build as _build
from . import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "_mla_decode_timeline.so")
CTA_WORDS, MAX_CTAS = 1024, 160
ROLE_BASE = {"softmax": 2, "mma": 402, "k": 802, "q": 914, "v": 924}
ROLE_CAP = {"softmax": 400, "mma": 400, "k": 112, "q": 10, "v": 100}
EV = dict(setup=1, chunk=2, sfull=4, pposted=5, ofull=6, epidone=7, exit=8, cluster_up=9, mma_qfull=10,
          mma_kfull=11, mma_pvgo=12, announced=15, first_tile=17, kload=16, qload=18, tile_loaded=19, vload=20,
          vtail_landed=21, vtail_done=22, conv_start=23, conv_done=24,
          conv_raw=25, v_landed=26, v_kconv=27)


def build_timeline_lib(force: bool = False) -> str:
    """Compile the instrumented copy (same sources, -DMLA_TIMELINE) next to the product library."""
    return _build.build(force=force, extra=["-DMLA_TIMELINE"], out=LIB)


def load_timeline_lib() -> ctypes.CDLL:
    lib = _lib.bind(build_timeline_lib())
    lib.mla_timeline_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    lib.mla_timeline_read.restype = ctypes.c_int
    return lib


def record(lib, p: W.Problem, launches: int = 6):
    """Runs the decode of problem `p` `launches` times; returns (events of the last split-KV
    launch [MAX_CTAS, CTA_WORDS] uint32, its event-timed duration in us, grid size)."""
    import torch

    import mla_decode_attention_12_b200 as mla

    dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
    q = torch.from_numpy(p.q.view(np.int16)).view(dt).cuda()
    kv = (torch.from_numpy(p.kvcache) if p.fp8_kv else torch.from_numpy(p.kvcache.view(np.int16)).view(dt)).cuda()
    bt = torch.from_numpy(p.block_table).cuda()
    sl = torch.from_numpy(p.cache_seqlens).cuda()
    rows = p.s_q * p.h_q
    parts = mla.num_sm_parts()
    sparse = p.indices is not None  # the token-level sparse decode: its own schedule and entry lists
    tokens = p.batch * p.s_q
    n_md, n_ns = mla.metadata_sizes(tokens if sparse else p.batch, p.h_q if sparse else rows, 1, parts)
    md = torch.zeros(parts, 8, dtype=torch.int32, device="cuda")
    ns = torch.zeros(n_ns, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    if sparse:
        _lib.check(lib.mla_get_metadata_sparse(tokens, p.indices.shape[2], p.h_q, 1, parts, md.data_ptr(),
                                               ns.data_ptr(), st), "mla_get_metadata_sparse")
    else:
        _lib.check(lib.mla_get_metadata(sl.data_ptr(), p.batch, rows, 1, parts, int(p.fp8_kv), md.data_ptr(),
                                        ns.data_ptr(), st),
                   "mla_get_metadata")
    ws_b, ws_s = (tokens, 1) if sparse else (p.batch, p.s_q)
    ws = torch.zeros(mla.workspace_bytes(ws_b, ws_s, p.h_q, 1, parts), dtype=torch.uint8, device="cuda")
    ind = torch.from_numpy(p.indices).cuda() if sparse else None
    call = mla.DecodeCall(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale, workspace=ws,
                          active_heads=p.active_heads, is_fp8_kvcache=p.fp8_kv, indices=ind)
    flush = torch.empty(2 * torch.cuda.get_device_properties(0).L2_cache_size, dtype=torch.uint8, device="cuda")
    us = []
    for _ in range(launches):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        _lib.check((lib.mla_decode_sparse_splitkv if sparse else lib.mla_decode_splitkv)(*call.args, st), "splitkv")
        e1.record()
        _lib.check(lib.mla_decode_combine(*call.combine_args, st), "mla_decode_combine")
        torch.cuda.synchronize()
        us.append(e0.elapsed_time(e1) * 1e3)
    status = ctypes.c_int(0)
    _lib.check(lib.mla_read_device_status(ws.data_ptr(), 1, ctypes.byref(status), st), "mla_read_device_status")
    assert status.value == 0, f"device status {status.value}"
    buf = np.zeros(MAX_CTAS * CTA_WORDS, np.uint32)
    _lib.check(lib.mla_timeline_read(buf.ctypes.data, buf.size), "mla_timeline_read")
    return buf.reshape(MAX_CTAS, CTA_WORDS), float(np.median(us[1:])), 2 * parts


def events(B, cta, role, t_off):
    """(ids, times in us on the common clock) of one role of one CTA."""
    lo, cap = ROLE_BASE[role], ROLE_CAP[role]
    x = B[cta, lo:lo + cap].astype(np.int64)
    x = x[x != 0]
    return x >> 27, (x & 0x7FFFFFF) / 1e3 + t_off[cta]


def phases(B, grid):
    """Per-CTA phase durations (us) of one launch."""
    start = B[:grid, 0].astype(np.int64) | (B[:grid, 1].astype(np.int64) << 32)
    t_off = (start - start.min()) / 1e3
    per = []
    for c in range(grid):
        i, t = events(B, c, "softmax", t_off)
        if not (i == EV["exit"]).any() or not (i == EV["sfull"]).any():
            continue
        im, tm = events(B, c - (c & 1), "mma", t_off)  # the pair's MMA warp runs in the even CTA
        q_full = tm[im == EV["mma_qfull"]]
        # chunks: split the softmax events at each chunk-begin
        begins = np.flatnonzero(i == EV["chunk"])
        chunks = []
        for a, b in zip(begins, list(begins[1:]) + [len(i)]):
            ii, tt = i[a:b], t[a:b]
            S, P = tt[ii == EV["sfull"]], tt[ii == EV["pposted"]]
            if len(S) == 0:
                continue
            chunks.append(dict(begin=tt[0], S=S, P=P, ofull=tt[ii == EV["ofull"]], epi=tt[ii == EV["epidone"]]))
        if not chunks:
            continue
        exit_t = t[i == EV["exit"]][-1]
        setup = t[i == EV["setup"]][0]
        stream = sum(ch["P"][-1] - ch["S"][0] for ch in chunks)
        pages = sum(len(ch["S"]) for ch in chunks)
        page_gaps = np.concatenate([np.diff(ch["P"]) for ch in chunks if len(ch["P"]) > 1] or [np.zeros(0)])
        trans, sub = [], []
        for a, b in zip(chunks[:-1], chunks[1:]):
            last_p = a["P"][-1]
            trans.append(b["S"][0] - last_p)
            of = a["ofull"][0] if len(a["ofull"]) else last_p
            ep = a["epi"][0] if len(a["epi"]) else of
            qf = q_full[q_full > last_p - 2.0]  # the next chunk's Q can be ready a little before the last P
            sub.append((of - last_p, ep - of, b["S"][0] - ep, (qf[0] - last_p) if len(qf) else np.nan))
        last = chunks[-1]
        per.append(dict(cta=c, entry=t_off[c], setup=setup - t_off[c], startup=chunks[0]["S"][0] - setup,
                        stream=stream, pages=pages, page_med=float(np.median(page_gaps)) if len(page_gaps) else np.nan,
                        chunks=len(chunks), trans=float(np.sum(trans)), trans_each=trans, trans_sub=sub,
                        last_epi=exit_t - last["P"][-1], exit=exit_t))
    end = max(r["exit"] for r in per)
    for r in per:
        r["idle_end"] = end - r["exit"]
    return per, end


def summarize(name: str, per, end: float, kernel_us: float) -> str:
    def col(key):
        return np.array([r[key] for r in per], float)

    def q(x):
        x = x[np.isfinite(x)]
        return f"{np.median(x):7.2f} | {np.percentile(x, 90):7.2f} | {x.max():7.2f}" if len(x) else "- | - | -"

    sub = np.array([s for r in per for s in r["trans_sub"]], float).reshape(-1, 4)
    each = np.array([x for r in per for x in r["trans_each"]], float)
    lines = [f"### {name}: split-KV {kernel_us:.1f} us (event-timed, median of the launches), last cluster exits at "
             f"{end:.1f} us after the first CTA starts",
             "",
             "| phase (per CTA) | median | p90 | max |",
             "|---|---|---|---|",
             f"| launch offset (entry after the first CTA's) | {q(col('entry'))} |",
             f"| set-up (barriers, tensor memory, grid dependency) | {q(col('setup'))} |",
             f"| start-up: set-up done -> first logits | {q(col('startup'))} |",
             f"| streaming (page loops) | {q(col('stream'))} |",
             f"| pages | {q(col('pages'))} |",
             f"| time per page (P to P) | {q(col('page_med'))} |",
             f"| chunks | {q(col('chunks'))} |",
             f"| transitions, sum per CTA | {q(col('trans'))} |",
             f"| last epilogue: last P -> exit | {q(col('last_epi'))} |",
             f"| idle at the end: exit -> last exit | {q(col('idle_end'))} |",
             f"| exit time | {q(col('exit'))} |"]
    if len(each):
        lines += [f"| one transition: last P -> next logits ({len(each)}) | {q(each)} |",
                  f"| .. wait for the last P V | {q(sub[:, 0])} |",
                  f"| .. output drained | {q(sub[:, 1])} |",
                  f"| .. then next logits | {q(sub[:, 2])} |",
                  f"| .. (MMA warp) next chunk's Q ready, after the last P | {q(sub[:, 3])} |"]
    return "\n".join(lines) + "\n"


def fp8_pipeline(B, grid) -> str:
    """The FP8 cache's K-stage cycle (converter warp 0 and the V producer of each CTA), per page:
    conversion, the wait for the other converter warps, the wait for a free V stage, the V copies
    until they land.  Empty when the record has no converter events (16-bit cache)."""
    start = B[:grid, 0].astype(np.int64) | (B[:grid, 1].astype(np.int64) << 32)
    t_off = (start - start.min()) / 1e3
    R = {k: [] for k in ("conversion (converter warp 0)", "rest of the converter warps", "wait for the V stage",
                         "V copies issued -> landed")}
    for c in range(grid):
        ik, tk = events(B, c, "k", t_off)
        st, dn = tk[ik == EV["conv_start"]], tk[ik == EV["conv_done"]]
        iv, tv = events(B, c, "v", t_off)
        kc, vl, vd = tv[iv == EV["v_kconv"]], tv[iv == EV["vload"]], tv[iv == EV["v_landed"]]
        n = min(len(st), len(dn), len(kc), len(vl), len(vd))
        if n == 0:
            continue
        R["conversion (converter warp 0)"] += list(dn[:n] - st[:n])
        R["rest of the converter warps"] += list(kc[:n] - dn[:n])
        R["wait for the V stage"] += list(vl[:n] - kc[:n])
        R["V copies issued -> landed"] += list(vd[:n] - vl[:n])
    if not R["conversion (converter warp 0)"]:
        return ""
    lines = ["| FP8 K-stage cycle, per page | p10 | median | p90 |", "|---|---|---|---|"]
    for k, v in R.items():
        v = np.array(v)
        lines.append(f"| {k} | {np.percentile(v, 10):6.2f} | {np.median(v):6.2f} | {np.percentile(v, 90):6.2f} |")
    return "\n".join(lines) + "\n"


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workloads", default="compute,spec_padded,long_split,fp16_norope,fp8_compute,sparse_fp8")
    ap.add_argument("--launches", type=int, default=6)
    ap.add_argument("--save", default=None, help="directory to save the raw event arrays (.npy) in")
    args = ap.parse_args(argv)
    import torch

    if not torch.cuda.is_available():
        raise SystemExit("the timeline needs a CUDA device")
    lib = load_timeline_lib()
    out = []
    for name in args.workloads.split(","):
        p = W.make_workload(name)
        B, us, grid = record(lib, p, args.launches)
        if args.save:
            os.makedirs(args.save, exist_ok=True)
            np.save(os.path.join(args.save, f"timeline_{name}.npy"), B)
        per, end = phases(B, grid)
        out.append(summarize(name, per, end, us) + fp8_pipeline(B, grid))
        print(out[-1], flush=True)
    return out


if __name__ == "__main__":
    sys.exit(0 if main() else 1)
