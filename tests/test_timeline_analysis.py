"""The timeline tool's phase split, on made-up event words (no GPU)."""
import numpy as np

from mla_decode_attention_12_b200 import timeline as T


def _word(ev, us):
    return (T.EV[ev] << 27) | int(round(us * 1e3))


def test_phase_split_of_a_two_chunk_cta():
    B = np.zeros((T.MAX_CTAS, T.CTA_WORDS), np.uint32)
    for c, start_ns in ((0, 1000), (1, 1500)):  # CTA 1 starts 0.5 us after CTA 0
        B[c, 0], B[c, 1] = start_ns, 0
        ev = [("setup", 2.0), ("chunk", 3.1)]
        t = 5.0
        for _ in range(3):  # chunk 0: 3 pages, 1 us apart
            ev += [("sfull", t), ("pposted", t + 0.6)]
            t += 1.0
        last_p = t - 0.4
        ev += [("ofull", last_p + 1.0), ("epidone", last_p + 3.0), ("chunk", last_p + 3.1)]
        t = last_p + 4.0  # next logits 4 us after the last P
        for _ in range(2):
            ev += [("sfull", t), ("pposted", t + 0.6)]
            t += 1.0
        ev += [("ofull", t), ("epidone", t + 2.0), ("exit", t + 2.5)]
        words = [_word(e, u) for e, u in ev]
        B[c, T.ROLE_BASE["softmax"]:T.ROLE_BASE["softmax"] + len(words)] = words
        if c == 0:  # the pair's MMA warp: the next chunk's Q ready 0.5 us after the last P
            B[c, T.ROLE_BASE["mma"]:T.ROLE_BASE["mma"] + 2] = [_word("mma_qfull", 4.5), _word("mma_qfull", last_p + 0.5)]
    per, end = T.phases(B, 2)
    assert len(per) == 2
    r = per[0]
    assert r["chunks"] == 2 and r["pages"] == 5
    assert abs(r["setup"] - 2.0) < 1e-9 and abs(r["startup"] - 3.0) < 1e-9
    assert abs(r["trans"] - 4.0) < 1e-9
    of, ep, nx, qr = r["trans_sub"][0]
    assert abs(of - 1.0) < 1e-9 and abs(ep - 2.0) < 1e-9 and abs(nx - 1.0) < 1e-9 and abs(qr - 0.5) < 1e-9
    assert abs(r["page_med"] - 1.0) < 1e-9
    # CTA 1 is the same schedule 0.5 us later: it exits last
    assert abs(per[1]["entry"] - 0.5) < 1e-9 and per[1]["idle_end"] == 0.0
    assert abs(per[0]["idle_end"] - 0.5) < 1e-9
    text = T.summarize("made-up", per, end, 20.0)
    assert "transitions" in text and "made-up" in text
