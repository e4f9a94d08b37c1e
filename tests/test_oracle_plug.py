"""Pins of the oracle's token plug ("Accelerating Sonar through speculation",
sections "MTP" and "MTP schedule for one token": the draft reads the target's
input tokens shifted one step left, and after verification a kernel plugs
the next target tokens into their positions, so the accepted count need not
reach the CPU first).  Hand-worked cases, written out from that definition."""
import numpy as np

ERR_TOKEN, ERR_CAPACITY = 1, 16


def test_mtp_one_token_accept_and_reject(orc):
    # k = 1: the target verified [t0, x0] = [7, 5]
    # accepted: emitted (x0, bonus 9); the draft next reads [x0, bonus]
    r = orc.plug_tokens([[7, 5]], [[5, 9]], [1])
    assert r["next"].tolist() == [[5, 9]] and r["err"] == 0
    # rejected: emitted (corrected 3); position 0 now holds 3, position 1 is
    # a don't-care pad (the drawn token again)
    r = orc.plug_tokens([[7, 5]], [[3, -1]], [0])
    assert r["next"].tolist() == [[3, 3]]


def test_k3_every_accept_length(orc):
    inp = [[10, 11, 12, 13]] * 4           # t0 = 10, drafts 11, 12, 13
    out = [[40, -1, -1, -1],               # n = 0: corrected 40
           [11, 41, -1, -1],               # n = 1
           [11, 12, 42, -1],               # n = 2
           [11, 12, 13, 43]]               # n = 3: bonus 43
    seq = np.full((4, 8), -7, np.int32)
    seq[:, :2] = [[1, 10]] * 4
    r = orc.plug_tokens(inp, out, [0, 1, 2, 3], seq, [2, 2, 2, 2])
    assert r["err"] == 0
    assert r["next"].tolist() == [[40, 12, 13, 40],
                                  [11, 41, 13, 41],
                                  [11, 12, 42, 42],
                                  [11, 12, 13, 43]]
    assert r["len"].tolist() == [3, 4, 5, 6]
    assert r["seq"][0].tolist() == [1, 10, 40, -7, -7, -7, -7, -7]
    assert r["seq"][3].tolist() == [1, 10, 11, 12, 13, 43, -7, -7]
    # invariant: the plugged prefix next[0..n] is exactly what was appended
    for b, n in enumerate([0, 1, 2, 3]):
        assert r["next"][b, :n + 1].tolist() == r["seq"][b, 2:3 + n].tolist()


def test_error_requests_and_capacity(orc):
    inp = [[1, 2, 3]] * 4
    out = [[2, 3, 9]] * 4
    seq = np.zeros((4, 5), np.int32)
    # b0: an upstream error (n = -1), skipped silently; b1: n = 5 > k, a
    # token error; b2: no room for 3 more tokens (len 3, capacity 5); b3: fine
    r = orc.plug_tokens(inp, out, [-1, 5, 2, 2], seq, [0, 0, 3, 2])
    assert r["err"] == ERR_TOKEN | ERR_CAPACITY
    assert r["next"][0].tolist() == [-1, -1, -1] and r["next"][1].tolist() == [-1, -1, -1]
    assert r["next"][2].tolist() == [2, 3, 9]  # next is still plugged
    assert r["len"].tolist() == [0, 0, 3, 5]
    assert r["seq"][2].tolist() == [0, 0, 0, 0, 0]
    assert r["seq"][3].tolist() == [0, 0, 2, 3, 9]
    # a negative length is a capacity error too
    r = orc.plug_tokens([[1, 2]], [[2, 4]], [1], np.zeros((1, 4), np.int32), [-1])
    assert r["err"] == ERR_CAPACITY and r["len"].tolist() == [-1]


def test_next_only_and_seq_only(orc):
    r = orc.plug_tokens([[5, 6, 7]], [[6, 1, -1]], [1], want_next=False,
                        seq_tokens=np.zeros((1, 4), np.int32), seq_len=[1])
    assert r["next"] is None and r["seq"][0].tolist() == [0, 6, 1, 0] and r["len"][0] == 3
    r = orc.plug_tokens([[5, 6, 7]], [[6, 1, -1]], [1])
    assert r["seq"] is None and r["next"].tolist() == [[6, 1, 1]]
