"""GPU parity of the denoising-loop driver against the oracle's schedule:
plan steps output dense attention, reused steps sparse attention on the
cached metadata plus the cached residual, over steps whose Q, K, V drift."""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import assert_out_close, dev_bf16, host

pytestmark = pytest.mark.gpu

# fidelity numbers are rel-L2 of bf16 outputs; both sides' rounding moves them
# by about 2^-9 / sqrt(3) relative, so they agree to a few 1e-3
FIDELITY_ABS = 5e-3


@pytest.mark.parametrize("steps,plan_steps", [(2, (1,)), (4, (1, 3))])
def test_schedule_matches_oracle(steps, plan_steps):
    w = synth.workload(1).with_(steps=steps, plan_steps=plan_steps)
    per_step = [synth.layer_tensors(w, step=t) for t in range(1, steps + 1)]
    sch = mcs.Schedule(w.G, w.k, plan_steps)
    got = []
    for t, (Q, K, V) in enumerate(per_step, start=1):
        q, k, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
        O, kind = sch.step(t, q, k, v)
        d = mcs.dense(q, k, v)
        rel, rel_nr = mcs.fidelity(O, d, sch.meta.residual)
        got.append((kind, host(O), rel, rel_nr))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    refs = [orc.schedule_head([(Q[0, h], K[0, h], V[0, h]) for Q, K, V in per_step], plan_steps,
                              w.G, w.k, w.scale) for h in range(w.H)]
    for h, ref in enumerate(refs):
        for t in range(steps):
            kind, O, _, _ = got[t]
            assert kind == ref[t]["kind"]
            assert_out_close(O[0, h], ref[t]["O"], f"step {t + 1} h{h}")
    # layer-wide fidelity against the oracle's (squared errors summed over heads)
    for t in range(steps):
        den = sum(float(np.sum(ref[t]["O_dense"] ** 2)) for ref in refs)
        num = sum(ref[t]["rel_l2"] ** 2 * float(np.sum(ref[t]["O_dense"] ** 2)) for ref in refs)
        num_nr = sum(ref[t]["rel_l2_no_residual"] ** 2 * float(np.sum(ref[t]["O_dense"] ** 2)) for ref in refs)
        _, _, rel, rel_nr = got[t]
        assert abs(rel - np.sqrt(num / den)) <= FIDELITY_ABS, (t + 1, rel, np.sqrt(num / den))
        assert abs(rel_nr - np.sqrt(num_nr / den)) <= FIDELITY_ABS, (t + 1, rel_nr, np.sqrt(num_nr / den))

def test_schedule_reuses_buffers_and_replans_on_shape_change():
    w = synth.workload(1)
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w))
    sch = mcs.Schedule(w.G, w.k, (1,))
    O1, k1 = sch.step(1, Q, K, V)
    O2, k2 = sch.step(2, Q, K, V)
    assert (k1, k2) == ("plan", "reused") and O1.data_ptr() == O2.data_ptr()
    # a smaller layer: new buffers, and its first step plans again
    O3, k3 = sch.step(3, Q[:, :1].contiguous(), K[:, :1].contiguous(), V[:, :1].contiguous())
    torch.cuda.synchronize()
    assert k3 == "plan" and O3.shape[1] == 1
    assert mcs.last_device_status() == 0


def test_saved_metadata_resumes_bit_for_bit(tmp_path):
    """Checkpoint and resume of the cached state: a reused step on metadata
    saved and loaded back equals the step on the original, bit for bit."""
    w = synth.workload("tiny")
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w))
    meta = mcs.plan(Q, K, V, w.G, w.k)
    O1 = mcs.sparse_step(Q, K, V, meta).clone()
    meta.save(tmp_path / "meta.pt")
    O2 = mcs.sparse_step(Q, K, V, mcs.Meta.load(tmp_path / "meta.pt"))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16))
