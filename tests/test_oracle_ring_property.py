"""The integer ring model (oracle/ring.py) against an independent, explicit model of
the buffer: per sequence, the list of committed-but-unfolded token indices and the
pending drafts, with the lazy flush rule (fold before appending n tokens when
len + n > W).  Random op sequences (hypothesis) must give the same counters after
every op, and the ring slots of the live entries must stay distinct: after a
verify (drafts pending, possibly after a fold in the same call) and again after
its commit.  Within each call, the slots it appends to must also avoid the
entries the call's own fold reads."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle.ring import MisuseError, RingModel


class ListModel:
    def __init__(self, B, W, K):
        self.W, self.R = W, W + max(K, 1)
        self.buf = [[] for _ in range(B)]       # committed, not folded
        self.drafts = [[] for _ in range(B)]    # pending
        self.seq = [0] * B
        self.ckpt = [0] * B
        self.flushes = [0] * B

    def _maybe_fold(self, b, n):
        if len(self.buf[b]) + n > self.W:
            self.ckpt[b] += len(self.buf[b])
            self.buf[b] = []
            self.flushes[b] += 1

    def decode(self):
        for b in range(len(self.seq)):
            self._maybe_fold(b, 1)
            self.buf[b].append(self.seq[b])
            self.seq[b] += 1

    def verify(self, K):
        for b in range(len(self.seq)):
            self._maybe_fold(b, K)
            self.drafts[b] = list(range(self.seq[b], self.seq[b] + K))

    def commit(self, a):
        for b in range(len(self.seq)):
            k = a[b] if 0 <= a[b] <= len(self.drafts[b]) else 0
            self.buf[b] += self.drafts[b][:k]
            self.seq[b] += k
            self.drafts[b] = []

    def flush(self):
        for b in range(len(self.seq)):
            if self.buf[b]:
                self.ckpt[b] += len(self.buf[b])
                self.buf[b] = []
                self.flushes[b] += 1


ops = st.lists(st.tuples(st.sampled_from(["decode", "verify", "flush"]), st.integers(1, 8),
                         st.lists(st.integers(-1, 9), min_size=3, max_size=3)), max_size=60)


def _check(rm, lm, W):
    """Counters equal, and the live entries (committed-but-unfolded plus pending
    drafts) are the explicit model's, each in its own ring slot."""
    assert rm.seq_pos.tolist() == lm.seq
    assert rm.ckpt_pos.tolist() == lm.ckpt
    assert rm.flush_count.tolist() == lm.flushes
    assert all(0 <= L <= W for L in rm.length.tolist())
    for b in range(len(lm.seq)):
        live = lm.buf[b] + lm.drafts[b]
        assert rm.live_entries(b) == live
        assert len({n % rm.R for n in live}) == len(live)  # no live entry shares a slot


def _check_call(rm, before, appended):
    """Within one call, the entries a fold reads (the committed entries before
    the call) and the slots the call appends to never coincide, fold or not."""
    for b in range(len(before)):
        touched = before[b] + appended[b]
        assert len({n % rm.R for n in touched}) == len(touched)


@settings(max_examples=200, deadline=None)
@given(W=st.integers(1, 12), K=st.integers(0, 8), seq=ops)
def test_ring_model_equals_explicit_buffer(W, K, seq):
    K = min(K, W)
    B = 3
    rm, lm = RingModel(B, W, K), ListModel(B, W, K)
    for op, k, acc in seq:
        before = [list(x) for x in lm.buf]
        if op == "decode":
            rm.decode()
            lm.decode()
            _check_call(rm, before, [[lm.seq[b] - 1] for b in range(B)])
        elif op == "flush":
            rm.flush()
            lm.flush()
        else:
            if K == 0:
                continue
            kk = min(k, K)
            rm.verify(kk)
            lm.verify(kk)
            _check_call(rm, before, lm.drafts)
            assert rm.pending.tolist() == [kk] * B
            _check(rm, lm, W)  # drafts pending, possibly after a fold in the same call
            bad = rm.commit(acc)
            lm.commit(acc)
            assert bad.tolist() == [not (0 <= a <= kk) for a in acc]
            assert rm.pending.tolist() == [0] * B
        _check(rm, lm, W)


def test_misuse_is_refused():
    rm = RingModel(2, 4, 2)
    rm.verify(2)
    for f in (rm.decode, rm.flush, lambda: rm.verify(1)):
        try:
            f()
            raise AssertionError("not refused")
        except MisuseError:
            pass
    rm.commit(np.array([1, 2]))
    try:
        rm.commit(np.array([0, 0]))
        raise AssertionError("not refused")
    except MisuseError:
        pass
