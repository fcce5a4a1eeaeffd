"""The seeded input generator (host logic, no method arithmetic): shapes, the k rule, bf16
rounding against PyTorch's own conversion, determinism and the structure each recipe plants."""
import numpy as np
import torch

from block_sparse_attention_blocks_b200 import workloads as W


def test_shapes_and_selection_rule():
    for name, w in W.WORKLOADS.items():
        T, Y, X = w.grid
        assert T * Y * X == w.N, name
        assert w.nb == -(-w.N // w.bs)
        assert w.d in (64, 128) and w.bs in (64, 128)
    assert W.get("wan14b_720p").nb == 591 and W.get("wan14b_720p").topk == 30   # 95 %
    assert W.get("wan1.3b_480p").nb == 256 and W.get("wan1.3b_480p").topk == 13
    assert W.get("hunyuan_720p").nb == 929 and W.get("hunyuan_720p").topk == 46
    sweep_k = sorted({k for k, _ in W.get("wan14b_720p").sweep})
    assert sweep_k == [30, 59, 118]                                            # 95/90/80 %


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0,
                                  3.0e38, 1e-40], np.float32)])            # ties to even, extremes
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = W.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16)
                          .float().numpy())


def test_generator_is_deterministic_and_seeded():
    w = W.get("pr1_1k")
    a = W.make_qkv(w)
    b = W.make_qkv(w, threads=1)
    c = W.make_qkv(w, seed=1)
    for x, y, z in zip(a, b, c):
        assert x.shape == (w.B, w.H, w.N, w.d) and x.dtype == np.uint16
        assert np.array_equal(x, y)
        assert not np.array_equal(x, z)


def test_recipes_plant_their_structure():
    w = W.get("pr1_1k")
    q, k, v = (W.bf16_bits_to_f32(t) for t in W.make_qkv(w))
    # the sink key of head 0 is amplified; head 1 has none
    norms = np.linalg.norm(k, axis=-1)
    assert norms[0, 0, 0] > 4 * np.median(norms[0, 0])
    assert norms[0, 1, 0] < 2 * np.median(norms[0, 1])
    # tokens of one cell share their centre: Q and K agree far more within a cell than V does
    cell = slice(0, 8)  # x = 0..7 of row y = 0, frame 0: one 8x8 cell
    qk = float(np.mean(q[0, 1, cell] @ k[0, 1, cell].T))
    vv = float(np.mean(v[0, 1, cell] @ v[0, 1, cell].T - np.diag(np.diag(v[0, 1, cell] @ v[0, 1, cell].T))))
    assert qk > 5.0 and abs(vv) < 2.0
