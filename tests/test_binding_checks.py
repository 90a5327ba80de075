"""The Python binding refuses buffers whose sizes differ from what the layer
and the metadata describe, before anything reaches the library (a mismatch
would be an out-of-bounds device access).  Host-only: CPU tensors stand in."""
import pytest
import torch

from sparse_attention_diffusion_mcs_b200 import api

CPU = torch.device("cpu")


def _meta(B=1, H=2, N=100, d=64, G=32, k=10):
    ng = -(-N // G)
    kk = min(k, N)
    return api.Meta(B, H, N, d, G, kk, ng, torch.zeros((B, H, N), dtype=torch.int32),
                    torch.zeros((B, H, ng, kk), dtype=torch.int32),
                    torch.zeros((B, H, N, d), dtype=torch.float32))


def test_matching_metadata_passes():
    api._check_meta(_meta(), 1, 2, 100, 64, CPU)
    api._check_meta(_meta(), 1, 2, 100, 64, CPU, G=32, k=10)
    api._check_meta(_meta(k=500), 1, 2, 100, 64, CPU, G=32, k=500)   # k clamped to N


@pytest.mark.parametrize("layer", [(1, 2, 101, 64), (1, 3, 100, 64), (2, 2, 100, 64), (1, 2, 100, 128)])
def test_metadata_for_another_layer_is_refused(layer):
    with pytest.raises(ValueError):
        api._check_meta(_meta(), *layer, CPU)


def test_metadata_for_another_group_size_or_k_is_refused():
    with pytest.raises(ValueError):
        api._check_meta(_meta(), 1, 2, 100, 64, CPU, G=64)
    with pytest.raises(ValueError):
        api._check_meta(_meta(), 1, 2, 100, 64, CPU, k=11)


def test_metadata_buffers_of_the_wrong_size_or_type_are_refused():
    m = _meta()
    m.kv_idx = torch.zeros((1, 2, 4, 9), dtype=torch.int32)           # one key short per group
    with pytest.raises(ValueError):
        api._check_meta(m, 1, 2, 100, 64, CPU)
    m = _meta()
    m.residual = torch.zeros((1, 2, 100, 64), dtype=torch.float64)    # wrong dtype
    with pytest.raises(ValueError):
        api._check_meta(m, 1, 2, 100, 64, CPU)
    m = _meta()
    m.perm = torch.zeros((1, 2, 200), dtype=torch.int32)[:, :, ::2]   # not contiguous
    with pytest.raises(ValueError):
        api._check_meta(m, 1, 2, 100, 64, CPU)
    m = _meta()
    m.n_groups = 5
    with pytest.raises(ValueError):
        api._check_meta(m, 1, 2, 100, 64, CPU)


def test_output_buffers_are_checked():
    api._check_tensor(torch.empty((1, 2, 8, 4), dtype=torch.bfloat16), "out", (1, 2, 8, 4), torch.bfloat16, CPU)
    for bad in (torch.empty((1, 2, 8, 5), dtype=torch.bfloat16), torch.empty((1, 2, 8, 4), dtype=torch.float16),
                torch.empty((1, 2, 4, 8), dtype=torch.bfloat16).transpose(2, 3)):
        with pytest.raises(ValueError):
            api._check_tensor(bad, "out", (1, 2, 8, 4), torch.bfloat16, CPU)
    with pytest.raises(TypeError):
        api._check_tensor(None, "out", (1,), torch.int32, CPU)


def test_metadata_save_load_roundtrip(tmp_path):
    """The cached metadata is the state a denoising loop resumes from: a save
    and load gives back the same sizes and the same bits."""
    m = _meta(N=100, k=10)
    g = torch.Generator().manual_seed(0)
    m.perm = torch.randperm(100, generator=g).to(torch.int32).repeat(1, 2, 1).contiguous()
    m.kv_idx = torch.randint(0, 100, m.kv_idx.shape, generator=g, dtype=torch.int32)
    m.residual = torch.randn(m.residual.shape, generator=g)
    path = tmp_path / "meta.pt"
    m.save(path)
    r = api.Meta.load(path, device="cpu")
    assert (r.B, r.H, r.N, r.d, r.G, r.k, r.n_groups) == (m.B, m.H, m.N, m.d, m.G, m.k, m.n_groups)
    for name in ("perm", "kv_idx", "residual"):
        a, b = getattr(m, name), getattr(r, name)
        assert a.dtype == b.dtype and torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_metadata_load_refuses_other_files(tmp_path):
    path = tmp_path / "other.pt"
    torch.save({"x": torch.zeros(3)}, path)
    with pytest.raises(ValueError):
        api.Meta.load(path, device="cpu")
