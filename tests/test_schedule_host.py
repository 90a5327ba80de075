"""Host-side sequencing of the denoising-loop driver, with the library calls
replaced by recorders (no GPU): which steps plan, which reuse, and when the
buffers are made."""
import torch

from sparse_attention_diffusion_mcs_b200 import denoise


class _Rec:
    def __init__(self, monkeypatch):
        self.calls = []
        monkeypatch.setattr(denoise.api, "alloc_workspace", lambda *a, **k: self._note("ws", torch.empty(1)))
        monkeypatch.setattr(denoise.api.Meta, "empty", staticmethod(lambda *a, **k: self._note("meta", object())))
        monkeypatch.setattr(denoise.api, "plan", lambda *a, **k: self.calls.append(("plan", k["meta"], k["out_dense"])))
        monkeypatch.setattr(denoise.api, "sparse_step", lambda Q, K, V, meta, scale, out: self.calls.append(("step", meta, out)))

    def _note(self, what, obj):
        self.calls.append((what,))
        return obj


def _qkv(h=2):
    t = torch.empty(1, h, 8, 4)
    return t, t, t


def test_plans_on_plan_steps_and_reuses_between(monkeypatch):
    rec = _Rec(monkeypatch)
    sch = denoise.Schedule(G=4, k=2, plan_steps=(1, 4))
    kinds = [sch.step(t, *_qkv())[1] for t in range(1, 7)]
    assert kinds == ["plan", "reused", "reused", "plan", "reused", "reused"]
    made = [c[0] for c in rec.calls if c[0] in ("ws", "meta")]
    assert made == ["ws", "meta"]                      # buffers made once
    metas = {id(c[1]) for c in rec.calls if c[0] in ("plan", "step")}
    outs = {id(c[2]) for c in rec.calls if c[0] in ("plan", "step")}
    assert len(metas) == 1 and len(outs) == 1         # and reused by every step


def test_first_step_plans_even_if_not_listed_and_reset_forces_a_plan(monkeypatch):
    _Rec(monkeypatch)
    sch = denoise.Schedule(G=4, k=2, plan_steps=(3,))
    assert [sch.step(t, *_qkv())[1] for t in (1, 2)] == ["plan", "reused"]
    sch.reset()
    assert sch.step(3, *_qkv())[1] == "plan" and sch.step(4, *_qkv())[1] == "reused"


def test_shape_change_makes_new_buffers_and_plans(monkeypatch):
    rec = _Rec(monkeypatch)
    sch = denoise.Schedule(G=4, k=2, plan_steps=(1,))
    sch.step(1, *_qkv(2))
    sch.step(2, *_qkv(2))
    assert sch.step(3, *_qkv(3))[1] == "plan"
    assert [c[0] for c in rec.calls if c[0] in ("ws", "meta")] == ["ws", "meta", "ws", "meta"]


def test_fidelity_closed_forms():
    D = torch.tensor([[[[3.0, 4.0], [0.0, 0.0]]]])          # ||D|| = 5
    R = torch.tensor([[[[1.0, 0.0], [0.0, 2.0]]]])
    O = (D + torch.tensor([[[[0.0, 0.5], [0.0, 0.0]]]])).to(torch.bfloat16)
    rel, rel_nr = denoise.fidelity(O, D.to(torch.bfloat16), R)
    assert abs(rel - 0.1) < 1e-12                            # ||(0, .5)|| / 5
    assert abs(rel_nr - (0.25 + 1 + 4) ** 0.5 / 5) < 1e-12   # O - R - D = (-1, .5, 0, -2)
