"""The bench's byte count B(b, S) (the package's own accounting) against the oracle's and
against the byte sizes of the tensors a step reads."""
import pytest

import bandwidth_bound_b200 as mk
import oracle
import synth


@pytest.mark.parametrize("wname", sorted(synth.WORKLOADS))
def test_step_bytes_matches_oracle(wname):
    w = synth.WORKLOADS[wname]
    lens = w.context_lengths()
    assert mk.step_bytes(w.model, lens) == oracle.model_bytes(w.model, lens)
    assert mk.step_bytes(w.model, lens[:1]) == oracle.model_bytes(w.model, lens[:1])


def test_step_bytes_equals_tensor_nbytes():
    w = synth.WORKLOADS["tiny-b1"]
    m, lens = w.model, w.context_lengths()
    wts = synth.make_weights(m)
    nb = sum(t.numel() * t.element_size() for lw in wts["layers"] for t in lw.values())
    nb += wts["final_norm"].numel() * 2 + wts["lm_head"].numel() * 2 + w.batch * m.hidden * 2
    nb += sum(lens) * m.n_layers * 2 * m.n_kv_heads * m.head_dim * 2
    assert mk.step_bytes(m, lens) == nb
