"""Host-side planning of a decoder step (no GPU): the int32 index arrays every kernel of the step
reads, and the argument checks made before anything is launched."""
import numpy as np
import pytest

from invariant_deterministic_rmsnorm_b200 import binding, inputs
from invariant_deterministic_rmsnorm_b200.decoder import Decoder


def _planner(max_seqs=4, cap=512, decode_attention="split"):
    d = object.__new__(Decoder)  # the planner needs no device state
    d.s, d.max_seqs, d.cap, d.decode_attention = inputs.LLAMA3_8B_4L, max_seqs, cap, decode_attention
    d.length = np.zeros(max_seqs, np.int64)
    return d


def test_prefill_plan_positions_rows_and_tiles():
    d = _planner()
    d.length[2] = 100  # slot 2 already holds a 100-token prefix
    p = d._plan([0, 2, 3], [[1] * 130, [2] * 5, [3]], "prefill")
    assert p["T"] == 136 and not p["split"]
    assert p["pos"].tolist() == list(range(130)) + list(range(100, 105)) + [0]
    assert p["rows"].tolist() == list(range(130)) + [2 * 512 + q for q in range(100, 105)] + [3 * 512]
    assert p["last"].tolist() == [129, 134, 135]
    assert p["tiles"] == [0, 2, 3, 4]  # 128-row query tiles per sequence
    assert p["q_indptr"].tolist() == [0, 130, 135, 136]
    assert p["kv_base"].tolist() == [0, 1024, 1536] and p["pos0"].tolist() == [0, 100, 0]
    assert binding.prefill_tiles([1, 128, 129, 0, 256]) == [0, 1, 2, 4, 4, 6]


def test_decode_plan_is_chunk_aligned():
    d = _planner()
    d.length[:] = [7, 0, 300, 511]
    p = d._plan([0, 2, 3], [[5], [6], [7]], "decode")
    assert p["split"] and p["T"] == 3
    assert p["kv_indptr"].tolist() == [0, 1024, 1536, 2048]
    assert all(v % 256 == 0 for v in p["kv_indptr"])
    assert p["kv_len"].tolist() == [8, 301, 512]
    assert p["rows"].tolist() == [7, 1024 + 300, 1536 + 511]
    assert p["seq"].tolist() == [0, 1, 2]
    # decode through prefill attention plans query tiles instead
    q = _planner(decode_attention="prefill")
    q.length[:] = [7, 0, 300, 511]
    pq = q._plan([0, 2, 3], [[5], [6], [7]], "decode")
    assert not pq["split"] and pq["tiles"] == [0, 1, 2, 3] and pq["pos0"].tolist() == [7, 300, 511]


@pytest.mark.parametrize("slots,tokens,phase", [
    ([1, 0], [[1], [2]], "prefill"),       # slots not increasing
    ([0, 0], [[1], [2]], "prefill"),       # repeated slot
    ([4], [[1]], "prefill"),               # slot outside the cache
    ([0], [[]], "prefill"),                # no new token
    ([0], [[1, 2]], "decode"),             # decode takes one token
    ([0], [[1]], "sample"),                # unknown phase
    ([0], [[1] * 513], "prefill"),         # outgrows the slot
])
def test_plan_rejects_bad_steps(slots, tokens, phase):
    with pytest.raises(ValueError):
        _planner()._plan(slots, tokens, phase)
