"""The Python binding's argument handling without a GPU: every wrapper is run on CPU tensors
against a stand-in for the library (which records the call and returns SA_OK), so the shape,
dtype and device checks and the argument marshalling are exercised; nothing here computes."""
import types

import pytest
import torch

from block_sparse_attention_blocks_b200 import sparse_attn as s


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes"):
            return lambda *a: 512
        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(s, "lib", lib)

    def need(t, name, dtype, ndim):  # the real check minus "must be a CUDA tensor"
        if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
            raise ValueError(name)

    monkeypatch.setattr(s, "_need", need)
    monkeypatch.setattr(s, "_stream", lambda device: None)
    monkeypatch.setattr(s, "_workspace", lambda device: torch.empty(256, dtype=torch.uint8))
    monkeypatch.setattr(s, "_cuda_device",
                        lambda device: torch.device(device) if device is not None else torch.device("cpu"))
    return lib


B, H, N, d, bs = 1, 2, 300, 64, 128
NB = 3


def bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def test_block_path_wrappers(fake):
    q = bf(B, H, N, d)
    qp, kp = s.pool_blocks(q, q, bs)
    assert qp.shape == (B, H, NB, d)
    mask, idx, cnt = s.select_mask_topk_topp(qp, kp, 2, 0.9)
    assert idx.shape == (B, H, NB, NB) and cnt.shape == (B, H, NB)
    s.pool_select_topk_topp(q, q, bs, 2, 0.9)
    s.block_scores(qp, kp)
    s.select_from_logits(f32(B, H, NB, NB), 2, 0.9)
    s.static_mask([(1, 1, 0, 0)] * H, B, NB, device="cpu")
    s.block_sparse_attn_fwd(q, q, q, idx, cnt, bs)
    s.dense_attn_fwd(q, q, q)
    s.squad_attn_fwd(q, q, q, 100)
    names = [c[0] for c in fake.calls]
    assert names == ["sa_pool_blocks", "sa_select_mask_topk_topp", "sa_pool_select_topk_topp",
                     "sa_block_scores", "sa_select_from_logits", "sa_static_mask",
                     "sa_block_sparse_attn_fwd", "sa_dense_attn_fwd", "sa_squad_attn_fwd"]


def test_block_path_shape_errors(fake):
    q = bf(B, H, N, d)
    idx, cnt = i32(B, H, NB, NB), i32(B, H, NB)
    with pytest.raises(ValueError):
        s.block_sparse_attn_fwd(q, bf(B, H, N - 1, d), q, idx, cnt, bs)     # k of another length
    with pytest.raises(ValueError):
        s.block_sparse_attn_fwd(q, q, q, i32(B, H, NB - 1, NB - 1), i32(B, H, NB - 1), bs)
    with pytest.raises(ValueError):
        s.block_sparse_attn_fwd(q, q, q, idx, cnt, 64)                      # lists for bs 128
    with pytest.raises(ValueError):
        s.pool_blocks(q, q, bs, qp=f32(B, H, NB + 1, d))
    with pytest.raises(ValueError):
        s.select_mask_topk_topp(f32(B, H, NB, d), f32(B, H, NB + 1, d), 2, 0.9)
    with pytest.raises(ValueError):
        s.select_from_logits(f32(B, H, NB, NB + 1), 2, 0.9)
    with pytest.raises(ValueError):
        s.block_scores(f32(B, H, NB, d), f32(B, H, NB, d), logits=f32(B, H, NB, NB - 1))
    with pytest.raises(ValueError):
        s.dense_attn_fwd(q, q, q, o=bf(B, H, N, d * 2))
    with pytest.raises(ValueError):
        s.squad_attn_fwd(q, q, bf(B, H + 1, N, d), 100)
    assert not fake.calls


def test_cluster_path_wrappers_and_errors(fake):
    q = bf(B, H, N, d)
    Cq, Ck = 5, 7
    assign, perm, cs, cz = s.kmeans(q, f32(B, H, Cq, d), 2)
    assert assign.shape == (B, H, N) and cz.shape == (B, H, Cq)
    s.cluster_sort(assign, Cq)
    sel = s.centroid_topp(f32(B, H, Cq, d), f32(B, H, Ck, d), i32(B, H, Ck), 0.9)
    assert sel.shape == (B, H, Cq, Ck)
    s.cluster_attn_fwd(q, q, q, i32(B, H, N), i32(B, H, N), sel)
    o, sel2 = s.svg2_attn_fwd(q, q, q, f32(B, H, Cq, d), f32(B, H, Ck, d), 2, 0.9)
    assert o.shape == q.shape and sel2.shape == (B, H, Cq, Ck)
    names = [c[0] for c in fake.calls]
    assert names == ["sa_kmeans", "sa_cluster_sort", "sa_centroid_topp", "sa_cluster_attn_fwd",
                     "sa_svg2_attn_fwd"]
    with pytest.raises(ValueError):
        s.kmeans(q, f32(B, H, Cq, d + 1), 2)
    with pytest.raises(ValueError):
        s.centroid_topp(f32(B, H, Cq, d), f32(B, H, Ck, d), i32(B, H, Ck + 1), 0.9)
    with pytest.raises(ValueError):
        s.cluster_attn_fwd(q, q, q, i32(B, H, N - 1), i32(B, H, N), sel)
    with pytest.raises(ValueError):
        s.cluster_attn_fwd(q, q, q, i32(B, H, N), i32(B, H, N), torch.zeros(B, H + 1, Cq, Ck, dtype=torch.uint8))
    with pytest.raises(ValueError):
        s.svg2_attn_fwd(q, q, q, f32(B, H, Cq, d), f32(B, H, Ck, d), 2, 0.9,
                        sel=torch.zeros(B, H, Cq, Ck + 1, dtype=torch.uint8))
    assert len(fake.calls) == 5
